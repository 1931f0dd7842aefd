// Causal flash attention for sm_100a: forward and backward on tcgen05 tensor cores.
//
// softmax(Q K^T / sqrt(hd) + causal mask) V  ("nanoGPT" wiki page, CausalSelfAttention:
// the explicit mask blocks attention to future tokens), computed tile by tile with an
// online softmax so the T x T score matrix never leaves the SM.
//
// Layout: q, k, v live in one bf16 buffer [B*T, 3, H, hdp] (hdp = head dim padded to 64 or
// 128, padding zero); each (b, h) slice is read with 3-D TMA boxes {64 features, rows, 1}
// under 128-byte swizzle, so rows past the end of a sequence arrive as zeros.
//
// Forward (one CTA per pair of 128-query tiles of one (b, h); heaviest causal pairs first):
//   warp 0      TMA: the two Q tiles once, then K_j and V_j through a ring of 5 (hd 128) or 8
//               (hd 64) slots, so that the loads run two blocks ahead of the products
//   warp 1      one thread alternates between the two tiles: O += P_j V_j (P from tensor memory,
//               V from shared memory), then S_{j+1} = Q K_{j+1}^T into that tile's TMEM scores,
//               so the tensor core works on one tile while the other tile's softmax runs
//   warps 2, 3  idle (they give their registers to the softmax warpgroups with setmaxnreg)
//   warps 4..11 two softmax warpgroups, one per query tile, one query row per thread holding its
//               128 scores: row max and sum in registers, P = exp2(...) (ex2.approx) as bf16
//               over the first 64 score columns (already read), where it is the A operand of the
//               PV product; O is rescaled in TMEM only when the running max grows
//               by more than 2^8 (otherwise the stale max stays exact because O and l use the
//               same one)
// Backward: delta = rowsum(dO * O) (kernels.cu), then two persistent kernels (one CTA per SM,
// walking (tile, head) items heaviest first):
//   dK/dV kernel: per 128-key tile, stepping over 128-query blocks from the diagonal:
//               S^T = K Q^T and dP^T = V dO^T into TMEM; elementwise warps write P^T and dS^T
//               back over them as bf16, the tensor-memory A operands of dV += P^T dO and
//               dK += dS^T Q (accumulating in TMEM)
//   dQ kernel:  per 128-query tile, stepping over 128-key blocks up to the diagonal:
//               S = Q K^T and dP = dO V^T into TMEM; dS as bf16 into a TMEM buffer, the A
//               operand of dQ += dS K
// Both are deterministic (no atomics).  Every wait is bounded (see ptx.cuh).
#include <algorithm>
#include <cmath>

#include "host.cuh"
#include "kernels.cuh"

namespace gptk {

static constexpr float kLog2e = 1.4426950408889634f;


// ====================================================================== forward
// One CTA per (b, h, pair of 128-query tiles A = 2p, B = 2p+1): two softmax warpgroups, one
// per query tile, and one MMA thread that alternates between them, so that the tensor core
// computes one tile's S or PV while the other tile's softmax runs.  K and V tiles stream
// through one ring shared by both query tiles (K_0, V_0, K_1, V_1, ...).
// TMEM: S_A [0,128), S_B [128,256), O_A [256,256+HD), O_B [384,384+HD).  P_t (bf16, two keys
// per column) goes over columns [0, 64) of S_t once the softmax holds the scores in registers;
// the next S_t product is issued only after the PV product that reads P_t has completed.
// Warpgroup 0 (TMA warp, MMA warp, two idle warps) gives registers to the two softmax
// warpgroups, so that each softmax thread holds its row's 128 scores at once.

template <int HD>
struct FwdSmem {
  static constexpr int TILE = HD * 256;         // 128 rows x HD bf16
  static constexpr int NS = HD == 128 ? 5 : 8;  // K/V ring slots
  static constexpr int Q0 = 0;                  // Q_A, Q_B
  static constexpr int KV = 2 * TILE;           // NS ring slots
  static constexpr int BAR = KV + NS * TILE;
  static constexpr int BYTES = BAR + 256 + 1024;
};

constexpr int kFwdThreads = 384;
constexpr int kFwdRegs = 168;          // per thread at launch: 65536 / 384, rounded down to 8
constexpr int kFwdRegsProducer = 80;   // warpgroup 0 after setmaxnreg.dec
constexpr int kFwdRegsSoftmax = 208;  // warpgroups 1, 2 after setmaxnreg.inc
static_assert(128 * kFwdRegsProducer + 256 * kFwdRegsSoftmax <= kFwdThreads * kFwdRegs,
              "the register split must fit the registers the block is launched with");

template <int HD>
__global__ void __launch_bounds__(kFwdThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_qkv, const AttnShape s, __nv_bfloat16* __restrict__ o,
                    long long ldo, float* __restrict__ lse_out, float scale_log2, unsigned int* __restrict__ amax_bits,
                    DevCtl ctl) {
  using L = FwdSmem<HD>;
  constexpr int NS = L::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;         // [NS]
  uint64_t* kv_empty = kv_full + NS;    // [NS]
  uint64_t* s_full = kv_empty + NS;     // [2] (A, B)
  uint64_t* p_full = s_full + 2;        // [2]
  uint64_t* o_done = s_full + 4;        // [2]
  uint64_t* drain = s_full + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 7);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_pairs = gridDim.y;
  const int pr = n_pairs - 1 - blockIdx.y;  // heaviest first
  const int bh = blockIdx.x;
  const int b = bh / s.H, h = bh % s.H;
  const int q0 = pr * 256;
  // KV blocks of each query tile t: [lo_t, 2 pr + t] (the diagonal block last; the lower end is 0,
  // or the block of the tile's first query minus the left window).  The ring streams blocks
  // jlo .. jlo + n_kv - 1, jlo = lo_A; tile t takes ring blocks f[t] .. f[t] + c[t] - 1.
  // c[1] = 0 when tile B lies past the end of the sequence.
  const int lo_a = s.win >= 0 ? max(0, (q0 - s.win) / 128) : 0;
  const int lo_b = s.win >= 0 ? max(0, (q0 + 128 - s.win) / 128) : 0;
  const int jlo = lo_a;
  const int c_t[2] = {2 * pr + 1 - lo_a, (q0 + 128 < s.T) ? 2 * pr + 2 - lo_b : 0};
  const int f_t[2] = {0, lo_b - lo_a};
  const int n_kv = c_t[1] > 0 ? f_t[1] + c_t[1] : c_t[0];
  constexpr int NCH = HD / 64;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_qkv);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  pdl_wait();  // q, k, v (and dO, lse, delta) come from the kernels before this one

  const int colq = h * s.hdp;
  const int colk = s.H * s.hdp + h * s.hdp;
  const int colv = 2 * s.H * s.hdp + h * s.hdp;

  if (warp < 4) {
    setmaxnreg_dec<kFwdRegsProducer>();
  if (warp == 0 && lane == 0) {
    // ---------------------------------------------- TMA producer
    bool ok = true;
    mbar_expect_tx(q_full, 2 * L::TILE);
    for (int t = 0; t < 2; ++t)
      for (int c = 0; c < NCH; ++c)
        tma_load_3d(sm + L::Q0 + t * L::TILE + c * 16384, &tm_qkv, q_full, colq + 64 * c, q0 + 128 * t, b);
    int issued = -1;
    for (int seq = 0; seq < 2 * n_kv && ok; ++seq) {
      const int slot = seq % NS;
      const uint32_t ph = (seq / NS) & 1;
      if (!mbar_wait(&kv_empty[slot], ph ^ 1u, ctl, abort_flag, 20)) { ok = false; break; }
      mbar_expect_tx(&kv_full[slot], L::TILE);
      const int col = (seq & 1) ? colv : colk;
      for (int c = 0; c < NCH; ++c)
        tma_load_3d(sm + L::KV + slot * L::TILE + c * 16384, &tm_qkv, &kv_full[slot], col + 64 * c,
                    (jlo + (seq >> 1)) * 128, b);
      issued = seq;
    }
    if (!ok) {
      volatile int never = 0;
      mbar_wait(q_full, 0, ctl, &never, 22);
      for (int seq = (issued >= NS ? issued - NS + 1 : 0); seq <= issued && issued >= 0; ++seq)
        mbar_wait(&kv_full[seq % NS], (seq / NS) & 1, ctl, &never, 22);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------- MMA issuer
    constexpr uint32_t idesc_s = idesc_bf16(128, 128, 0, 0);
    constexpr uint32_t idesc_o = idesc_bf16(128, HD, 0, 1);
    bool ok = mbar_wait(q_full, 0, ctl, abort_flag, 23);
    bool issued = false;
    auto kv_wait = [&](int seq) -> bool {
      return mbar_wait(&kv_full[seq % NS], (seq / NS) & 1, ctl, abort_flag, 24);
    };
    // operand descriptors computed once; the MMAs of a product go out back to back (umma8_*)
    const uint64_t dQ0 = sdesc_sw128(smem_u32(sm + L::Q0), 16, 1024);
    const uint64_t dKV0 = sdesc_sw128(smem_u32(sm + L::KV), 16, 1024);     // K-major (K for S)
    const uint64_t dKVm0 = sdesc_sw128(smem_u32(sm + L::KV), 16384, 1024);  // MN-major (V for PV)
    auto issue_s = [&](int t, int j) {
      const uint64_t dQ = sdesc_add(dQ0, t * L::TILE);
      const uint64_t dK = sdesc_add(dKV0, ((2 * j) % NS) * L::TILE);
      if (HD == 128) {
        uint32_t dd[8];
        uint64_t aa[8], bb[8];
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          dd[kk] = tbase + 128 * t;
          aa[kk] = sdesc_add(dQ, off);
          bb[kk] = sdesc_add(dK, off);
        }
        umma8_ss(dd, aa, bb, idesc_s, 0xfeu);
      } else {
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_bf16(tbase + 128 * t, sdesc_add(dQ, off), sdesc_add(dK, off), idesc_s, kk > 0);
        }
      }
      umma_commit(&s_full[t]);
    };
    auto issue_pv = [&](int t, int j) {
      const uint64_t dV = sdesc_add(dKVm0, ((2 * j + 1) % NS) * L::TILE);
      uint32_t dd[8], aa[8];
      uint64_t bb[8];
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {  // keys 16 kk .. 16 kk + 15
        dd[kk] = tbase + 256 + 128 * t;
        aa[kk] = tbase + 128 * t + 8 * kk;
        bb[kk] = sdesc_add(dV, kk * 2048);
      }
      umma8_ts(dd, aa, bb, idesc_o, j == f_t[t] ? 0xfeu : 0xffu);
      umma_commit(&o_done[t]);
    };
    // ring block j (0-based from jlo): tile t computes S for it when f[t] <= j < f[t] + c[t]
    auto takes = [&](int t, int j) { return c_t[t] > 0 && j >= f_t[t] && j < f_t[t] + c_t[t]; };
    if (ok && kv_wait(0)) {
      tc_fence_after();
      for (int t = 0; t < 2; ++t)
        if (takes(t, 0)) issue_s(t, 0);
      umma_commit(&kv_empty[0]);
      issued = true;
    } else {
      ok = false;
    }
    for (int j = 0; j < n_kv && ok; ++j) {
      for (int t = 0; t < 2 && ok; ++t) {
        if (takes(t, j)) {
          if (!mbar_wait(&p_full[t], (j - f_t[t]) & 1, ctl, abort_flag, 26) || !kv_wait(2 * j + 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(t, j);
        }
        if (takes(t, j + 1)) {
          if (!kv_wait(2 * j + 2)) { ok = false; break; }
          // S_{j+1} overwrites the columns that hold P_j: the PV product must have read them
          if (takes(t, j) && !mbar_wait(&o_done[t], (j - f_t[t]) & 1, ctl, abort_flag, 25)) { ok = false; break; }
          tc_fence_after();
          issue_s(t, j + 1);
        }
      }
      if (!ok) break;
      umma_commit(&kv_empty[(2 * j + 1) % NS]);                   // V_j
      if (j + 1 < n_kv) umma_commit(&kv_empty[(2 * j + 2) % NS]);  // K_{j+1}
    }
    if (!ok && issued) {
      volatile int never = 0;
      umma_commit(drain);
      mbar_wait(drain, 0, ctl, &never, 28);
    }
  }
  } else {
    setmaxnreg_inc<kFwdRegsSoftmax>();
    // ---------------------------------------------- softmax: warpgroup 1 + t handles query tile t
    const int t = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int qi = q0 + 128 * t + r;
    const int n = c_t[t];
    const int jfirst = jlo + f_t[t];  // the tile's first KV block
    const int diag = 2 * pr + t;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tbase + 128 * t + lane_off;
    const uint32_t tO = tbase + 256 + 128 * t + lane_off;
    float m = -INFINITY, l = 0.f;
    bool ok = n > 0;
    for (int i = 0; i < n; ++i) {
      if (!mbar_wait(&s_full[t], i & 1, ctl, abort_flag, 29)) { ok = false; break; }
      tc_fence_after();
      const int j = jfirst + i;
      const int kbase = j * 128;
      // masked: the diagonal block (causal), or a block reaching below the window of the tile's
      // last query (keys before qi - win do not exist for query qi)
      const bool dg = (j == diag) || (s.win >= 0 && kbase < q0 + 128 * t + 127 - s.win);
      const int kmin = s.win >= 0 ? qi - s.win : 0;
      uint32_t raw[128];
      float* sv = reinterpret_cast<float*>(raw);
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32_nowait(tS + 32 * c, raw + 32 * c);
      tmem_wait_ld();
      tmem_fence_regs<128>(raw);
      if (dg) {
        // keys after the query, past the sequence or before the window do not exist
#pragma unroll
        for (int e = 0; e < 128; ++e) {
          const int key = kbase + e;
          if (key > qi || key >= s.T || key < kmin) sv[e] = -INFINITY;
        }
      }
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = -INFINITY;
#pragma unroll
      for (int e = 0; e < 128; e += 2) mx8[(e >> 1) & 7] = fmax3(mx8[(e >> 1) & 7], sv[e], sv[e + 1]);
      float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      mx *= scale_log2;  // -inf when every key of the block lies outside this row's window
      const float m_new = fmaxf(m, mx);
      float alpha = 1.f;
      if (m_new > m + 8.f) {
        alpha = ex2_approx(m - m_new);
        m = m_new;
      }
      // O is free here: the MMA thread issued this block's S product only after the tile's
      // previous P V product had completed, and s_full (a commit of every product issued before)
      // has been observed
      if (i > 0) {
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < HD / 32; ++c) {
            float ov[32];
            tmem_ld32(tO + c * 32, ov);
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] *= alpha;
            tmem_st32(tO + c * 32, ov);
          }
        }
      }
      // P = exp2(s * scale - m) as bf16 over score columns [0, 64) (masked scores are -inf and
      // give 0); a row with no visible key yet (m = -inf) takes 0 as its offset: its scores are
      // all -inf
      const float m_off = m == -INFINITY ? 0.f : m;
      const float2 sc2 = make_float2(scale_log2, scale_log2), nm2 = make_float2(-m_off, -m_off);
      float2 rs2[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) rs2[k] = make_float2(0.f, 0.f);
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        uint32_t pw[8];  // keys 16 g .. 16 g + 15, two per word
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int e = 16 * g + 2 * k;
          const float2 x = ffma2(make_float2(sv[e], sv[e + 1]), sc2, nm2);
          const float2 pv = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          rs2[k & 3] = fadd2(rs2[k & 3], pv);
          pw[k] = pack_bf16x2(pv.x, pv.y);
        }
        tmem_st8(tS + 8 * g, pw);
      }
      const float rs = ((rs2[0].x + rs2[0].y) + (rs2[1].x + rs2[1].y)) + ((rs2[2].x + rs2[2].y) + (rs2[3].x + rs2[3].y));
      l = l * alpha + rs;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
    }
    if (ok && mbar_wait(&o_done[t], (n - 1) & 1, ctl, abort_flag, 31)) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool row_ok = qi < s.T;
      __nv_bfloat16* orow = o + ((long long)b * s.T + qi) * ldo + (long long)h * s.hd;
      float am = 0.f;  // max |o| of the row (for an 8-bit cast of o)
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        float ov[32];
        tmem_ld32(tO + c * 32, ov);
#pragma unroll
        for (int e = 0; e < 32; ++e) ov[e] *= inv_l;
        if (amax_bits && row_ok) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (c * 32 + e < s.hd) am = fmaxf(am, fabsf(ov[e]));
        }
        if (row_ok) {
          if (s.hd == HD) {
            uint4* d = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int g = 0; g < 4; ++g)
              d[g] = make_uint4(pack_bf16x2(ov[8 * g], ov[8 * g + 1]), pack_bf16x2(ov[8 * g + 2], ov[8 * g + 3]),
                                pack_bf16x2(ov[8 * g + 4], ov[8 * g + 5]), pack_bf16x2(ov[8 * g + 6], ov[8 * g + 7]));
          } else {
            for (int e = 0; e < 32; ++e)
              if (c * 32 + e < s.hd) orow[c * 32 + e] = __float2bfloat16_rn(ov[e]);
          }
        }
      }
      if (row_ok) lse_out[(long long)bh * s.T + qi] = (m + log2f(l)) * 0.6931471805599453f;
      if (amax_bits) {
        // one atomic per warp; o is stored in bf16 and the rounding is monotonic
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, sh));
        if (lane == 0) atomicMax(amax_bits, __float_as_uint(__bfloat162float(__float2bfloat16_rn(am))));
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// The w-th item of CTA c in a grid of G CTAs: round r deals items r G .. r G + G - 1, to the
// CTAs in order on even rounds and in reverse on odd ones, so that every CTA gets a similar mix
// of the heavy and light items of a list sorted heaviest first.
__device__ __forceinline__ int zigzag_item(int r, int c, int G) { return r * G + ((r & 1) ? G - 1 - c : c); }

// ====================================================================== backward: dK, dV
// Persistent: one CTA per SM walks a list of (b, h, 128-key tile) items, heaviest tiles first,
// dealt to the CTAs in zigzag order; for each item it steps over 128-query blocks from the
// diagonal block on.
//   S^T = K Q^T and dP^T = V dO^T go into TMEM (M = 128 keys, N = 128 queries, full-rate MMAs).
//   Sixteen elementwise warps turn them into P^T = exp2(S^T scale - lse) and
//   dS^T = P^T (dP^T - delta) and write both back as bf16 over the fp32 columns each warp has
//   just read (element (key, query) at lane key, column query/2 of its 16-query group), where
//   they are the tensor-memory A operand of dV += P^T dO and dK += dS^T Q.
//   The block's queries go in two halves: the dV/dK products of the first half run while the
//   elementwise warps work on the second.
// TMEM: S^T/P^T [0,128), dP^T/dS^T [128,256), dV [256, 256+HD), dK [384, 384+HD).
// Across items nothing waits for a whole CTA to drain: the next item's K and V load as soon as
// the last S^T / dP^T products of the current one have read theirs, the query-block ring runs on
// without a break, and the next item's first S^T / dP^T products run while the elementwise
// warps write the current item's dK and dV out of TMEM.
// The per-query statistics (lse in log2 units, delta) of each block are staged in shared
// memory by the elementwise warps, loaded from global memory one block ahead.

constexpr int kBwdThreads = 576;  // TMA warp, MMA warp, 16 elementwise warps
constexpr int kBwdEw = 16;        // elementwise warps: 4 per TMEM lane quadrant

template <int HD>
struct DkvSmem {
  static constexpr int TILE = HD * 256;            // 128 rows x HD bf16 (64-column chunks of 16 KB)
  static constexpr int K = 0;
  static constexpr int V = K + TILE;
  static constexpr int Q0 = V + TILE;              // [2] query-block ring
  static constexpr int DO0 = Q0 + 2 * TILE;        // [2]
  static constexpr int STATS = DO0 + 2 * TILE;     // [2][lse2 x 128, delta x 128] fp32
  static constexpr int BAR = STATS + 2048;
  static constexpr int BYTES = BAR + 256 + 1024;
};

// The query blocks of key tile kt: from the diagonal block on, up to the last query whose window
// still reaches the tile's last key.
__device__ __forceinline__ int dkv_blocks(const AttnShape& s, int kt) {
  int n = (s.T + 127) / 128 - kt;
  if (s.win >= 0) n = min(n, (kt * 128 + 127 + s.win) / 128 - kt + 1);
  return n;
}

template <int HD>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tm_kv128, const __grid_constant__ CUtensorMap tm_q128,
                        const __grid_constant__ CUtensorMap tm_do128, const AttnShape s, const float* __restrict__ lse,
                        const float* __restrict__ delta, __nv_bfloat16* __restrict__ dqkv, float scale_log2,
                        float scale, DevCtl ctl) {
  using L = DkvSmem<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;     // [2]
  uint64_t* q_empty = bars + 3;    // [2]
  uint64_t* s_full = bars + 5;
  uint64_t* h_full = bars + 6;     // [2] one per half of the elementwise pass
  uint64_t* d_done = bars + 8;
  uint64_t* stats_bar = bars + 9;  // [2]
  uint64_t* acc_full = bars + 11;
  uint64_t* drain = bars + 12;
  uint64_t* kv_empty = bars + 13;
  uint64_t* acc_empty = bars + 14;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* stats = reinterpret_cast<float*>(sm + L::STATS);

  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_kt = (s.T + 127) / 128;
  const int BH = s.B * s.H;
  const int n_items = n_kt * BH;  // item w: key tile w / BH (heaviest first), head w % BH
  constexpr int NCH = HD / 64;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&h_full[i], kBwdEw);
      mbar_init(&stats_bar[i], kBwdEw);
    }
    mbar_init(s_full, 1);
    mbar_init(d_done, 1);
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kBwdEw);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  pdl_wait();  // q, k, v (and dO, lse, delta) come from the kernels before this one
  const uint32_t tS = tbase;
  const uint32_t tdP = tbase + 128;
  const uint32_t tdV = tbase + 256;
  const uint32_t tdK = tbase + 384;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA producer
    bool ok = true;
    int g = 0;                    // query blocks loaded, over all items
    int kv_issued = -1, issued_g = -1;
    for (int r = 0; ok; ++r) {
      const int w = zigzag_item(r, blockIdx.x, gridDim.x);
      if (w >= n_items) break;
      const int kt = w / BH, bh = w % BH;
      const int b = bh / s.H, h = bh % s.H;
      const int colk = s.H * s.hdp + h * s.hdp, colv = 2 * s.H * s.hdp + h * s.hdp;
      const int colq = h * s.hdp, cold = h * s.hdp;
      // K and V of the previous item are read by its S^T / dP^T products until kv_empty
      if (r > 0 && !mbar_wait(kv_empty, (r - 1) & 1, ctl, abort_flag, 40)) { ok = false; break; }
      mbar_expect_tx(kv_full, 2 * L::TILE);
      for (int c = 0; c < NCH; ++c) {
        tma_load_3d(sm + L::K + c * 16384, &tm_kv128, kv_full, colk + 64 * c, kt * 128, b);
        tma_load_3d(sm + L::V + c * 16384, &tm_kv128, kv_full, colv + 64 * c, kt * 128, b);
      }
      kv_issued = r;
      const int n_it = dkv_blocks(s, kt);
      for (int it = 0; it < n_it; ++it, ++g) {
        const int st = g & 1;
        if (!mbar_wait(&q_empty[st], ((g >> 1) & 1) ^ 1u, ctl, abort_flag, 40)) { ok = false; break; }
        const int qb = (kt + it) * 128;
        mbar_expect_tx(&q_full[st], 2 * L::TILE);
        for (int c = 0; c < NCH; ++c) {
          tma_load_3d(sm + L::Q0 + st * L::TILE + c * 16384, &tm_q128, &q_full[st], colq + 64 * c, qb, b);
          tma_load_3d(sm + L::DO0 + st * L::TILE + c * 16384, &tm_do128, &q_full[st], cold + 64 * c, qb, b);
        }
        issued_g = g;
      }
    }
    if (!ok) {
      // wait (bounded) for the copies still in flight before the CTA goes away
      volatile int never = 0;
      if (kv_issued >= 0) mbar_wait(kv_full, kv_issued & 1, ctl, &never, 41);
      for (int gg = (issued_g >= 1 ? issued_g - 1 : 0); gg <= issued_g && issued_g >= 0; ++gg)
        mbar_wait(&q_full[gg & 1], (gg >> 1) & 1, ctl, &never, 41);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_s = idesc_bf16(128, 128, 0, 0);
    constexpr uint32_t idesc_d = idesc_bf16(128, HD, 0, 1);
    bool ok = true;
    bool issued = false;
    // operand descriptors, computed once: K-major K, V, Q, dO; MN-major Q, dO for dK, dV
    const uint64_t dK = sdesc_sw128(smem_u32(sm + L::K), 16, 1024);
    const uint64_t dV = sdesc_sw128(smem_u32(sm + L::V), 16, 1024);
    uint64_t dQk[2], dDk[2], dQm[2], dDm[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      dQk[i] = sdesc_sw128(smem_u32(sm + L::Q0 + i * L::TILE), 16, 1024);
      dDk[i] = sdesc_sw128(smem_u32(sm + L::DO0 + i * L::TILE), 16, 1024);
      dQm[i] = sdesc_sw128(smem_u32(sm + L::Q0 + i * L::TILE), 16384, 1024);
      dDm[i] = sdesc_sw128(smem_u32(sm + L::DO0 + i * L::TILE), 16384, 1024);
    }
    int g = 0;
    for (int r = 0; ok; ++r) {
      const int w = zigzag_item(r, blockIdx.x, gridDim.x);
      if (w >= n_items) break;
      const int n_it = dkv_blocks(s, w / BH);
      if (!mbar_wait(kv_full, r & 1, ctl, abort_flag, 42)) { ok = false; break; }
      for (int it = 0; it < n_it && ok; ++it, ++g) {
        const int st = g & 1;
        if (!mbar_wait(&q_full[st], (g >> 1) & 1, ctl, abort_flag, 43)) { ok = false; break; }
        // the S^T / dP^T columns still hold the previous block's P^T / dS^T until its products finish
        if (g > 0 && !mbar_wait(d_done, (g - 1) & 1, ctl, abort_flag, 44)) { ok = false; break; }
        tc_fence_after();
        const uint64_t dQ = st ? dQk[1] : dQk[0], dD = st ? dDk[1] : dDk[0];
        const uint64_t dQn = st ? dQm[1] : dQm[0], dDn = st ? dDm[1] : dDm[0];
        // S^T and dP^T, interleaved, in groups of four K steps issued back to back
#pragma unroll
        for (int gq = 0; gq < HD / 64; ++gq) {
          uint32_t dd[8];
          uint64_t aa[8], bb[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t off = gq * 16384 + i * 32;
            dd[2 * i] = tS;
            dd[2 * i + 1] = tdP;
            aa[2 * i] = sdesc_add(dK, off);
            aa[2 * i + 1] = sdesc_add(dV, off);
            bb[2 * i] = sdesc_add(dQ, off);
            bb[2 * i + 1] = sdesc_add(dD, off);
          }
          umma8_ss(dd, aa, bb, idesc_s, gq == 0 ? 0xfcu : 0xffu);
        }
        umma_commit(s_full);
        if (it == n_it - 1) umma_commit(kv_empty);  // the item's K and V are no longer read
        issued = true;
        // dV and dK of the previous item are in TMEM until the elementwise warps have read them
        if (it == 0 && r > 0 && !mbar_wait(acc_empty, (r - 1) & 1, ctl, abort_flag, 48)) { ok = false; break; }
        for (int hh = 0; hh < 2 && ok; ++hh) {
          if (!mbar_wait(&h_full[hh], g & 1, ctl, abort_flag, 45)) { ok = false; break; }
          tc_fence_after();
          uint32_t dd[8], aa[8];
          uint64_t bb[8];
#pragma unroll
          for (int kq = 0; kq < 4; ++kq) {
            const int kk = 4 * hh + kq;  // 16 queries
            dd[2 * kq] = tdV;
            dd[2 * kq + 1] = tdK;
            aa[2 * kq] = tS + 16 * kk;
            aa[2 * kq + 1] = tdP + 16 * kk;
            bb[2 * kq] = sdesc_add(dDn, kk * 2048);
            bb[2 * kq + 1] = sdesc_add(dQn, kk * 2048);
          }
          umma8_ts(dd, aa, bb, idesc_d, (hh == 0 && it == 0) ? 0xfcu : 0xffu);
        }
        if (!ok) break;
        umma_commit(d_done);
        umma_commit(&q_empty[st]);
      }
      if (!ok) break;
      umma_commit(acc_full);
    }
    if (!ok && issued) {
      volatile int never = 0;
      umma_commit(drain);
      mbar_wait(drain, 0, ctl, &never, 46);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------ elementwise warps
    const int ew = warp - 2;         // 0..15
    const int quad = warp & 3;       // TMEM lane quadrant: keys 32 quad .. 32 quad + 31
    const int wq = ew >> 2;          // 16-query group within each half
    const int r_key = quad * 32 + lane;  // key row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    // statistics staging: this warp owns 8 queries of each block (lanes 0-7 lse, 8-15 delta)
    const int qq = 8 * ew + (lane & 7);
    auto stat_of = [&](int bh, int qb) -> float {
      const int q = qb + qq;
      if (lane >= 16 || q >= s.T) return 0.f;
      return lane < 8 ? __ldg(lse + (long long)bh * s.T + q) * kLog2e : __ldg(delta + (long long)bh * s.T + q);
    };
    // the block after (item r, block it): the next block of the item, else the next item's first
    auto next_block = [&](int r, int it, int n_it, int& bh_n, int& qb_n) -> bool {
      if (it + 1 < n_it) {
        const int w = zigzag_item(r, blockIdx.x, gridDim.x);
        bh_n = w % BH;
        qb_n = (w / BH + it + 1) * 128;
        return true;
      }
      const int w = zigzag_item(r + 1, blockIdx.x, gridDim.x);
      if (w >= n_items) return false;
      bh_n = w % BH;
      qb_n = (w / BH) * 128;
      return true;
    };
    bool ok = true;
    int g = 0;
    float v_next = 0.f;
    {
      const int w0 = zigzag_item(0, blockIdx.x, gridDim.x);
      if (w0 < n_items) v_next = stat_of(w0 % BH, (w0 / BH) * 128);
    }
    for (int r = 0; ok; ++r) {
      const int w = zigzag_item(r, blockIdx.x, gridDim.x);
      if (w >= n_items) break;
      const int kt = w / BH, bh = w % BH;
      const int b = bh / s.H, h = bh % s.H;
      const int k0 = kt * 128;
      const int key = k0 + r_key;
      const int n_it = dkv_blocks(s, kt);
      for (int it = 0; it < n_it; ++it, ++g) {
        const int st = g & 1;
        const int qb = (kt + it) * 128;
        if (lane < 16) stats[st * 256 + (lane < 8 ? 0 : 128) + qq] = v_next;
        __syncwarp();
        if (lane == 0) mbar_arrive(&stats_bar[st]);
        int bh_n, qb_n;
        if (next_block(r, it, n_it, bh_n, qb_n)) v_next = stat_of(bh_n, qb_n);  // one block ahead
        if (!mbar_wait(&stats_bar[st], (g >> 1) & 1, ctl, abort_flag, 50)) { ok = false; break; }
        if (!mbar_wait(s_full, g & 1, ctl, abort_flag, 47)) { ok = false; break; }
        tc_fence_after();
        // the diagonal block, the ragged end, or a block whose last query's window misses the
        // tile's first key
        const bool masked = (it == 0) || (qb + 128 > s.T) || (s.win >= 0 && qb + 127 - s.win > k0);
        for (int hh = 0; hh < 2; ++hh) {
          const int c = 4 * hh + wq;  // queries qb + 16c .. qb + 16c + 15
          uint32_t rs[16], rd[16];
          tmem_ld16_nowait(tS + lane_off + 16 * c, rs);
          tmem_ld16_nowait(tdP + lane_off + 16 * c, rd);
          tmem_wait_ld();
          tmem_fence_regs<16>(rs);
          tmem_fence_regs<16>(rd);
          const float* stl = stats + st * 256 + 16 * c;
          uint32_t pw[8], dw[8];
#pragma unroll
          for (int gg = 0; gg < 4; ++gg) {
            const float4 l4 = *reinterpret_cast<const float4*>(stl + 4 * gg);
            const float4 d4 = *reinterpret_cast<const float4*>(stl + 128 + 4 * gg);
            const float l2[4] = {l4.x, l4.y, l4.z, l4.w};
            const float dl[4] = {d4.x, d4.y, d4.z, d4.w};
            float p[4], ds[4];
            if (masked) {  // the diagonal block or the ragged end: causal / range mask
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int e = 4 * gg + k;
                const int q = qb + 16 * c + e;
                float pv = ex2_approx(fmaf(__uint_as_float(rs[e]), scale_log2, -l2[k]));
                if (q < key || q >= s.T || (s.win >= 0 && q - s.win > key)) pv = 0.f;
                p[k] = pv;
                ds[k] = pv * (__uint_as_float(rd[e]) - dl[k]);
              }
            } else {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int e = 4 * gg + k;
                p[k] = ex2_approx(fmaf(__uint_as_float(rs[e]), scale_log2, -l2[k]));
                ds[k] = p[k] * (__uint_as_float(rd[e]) - dl[k]);
              }
            }
            pw[2 * gg] = pack_bf16x2(p[0], p[1]);
            pw[2 * gg + 1] = pack_bf16x2(p[2], p[3]);
            dw[2 * gg] = pack_bf16x2(ds[0], ds[1]);
            dw[2 * gg + 1] = pack_bf16x2(ds[2], ds[3]);
          }
          // bf16 P^T and dS^T over the first 8 of the 16 columns this warp has just read
          tmem_st8(tS + lane_off + 16 * c, pw);
          tmem_st8(tdP + lane_off + 16 * c, dw);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&h_full[hh]);
        }
      }
      if (!ok) break;
      // epilogue: the four warps of a quadrant split dK (times the softmax scale) and dV
      if (!mbar_wait(acc_full, r & 1, ctl, abort_flag, 49)) { ok = false; break; }
      tc_fence_after();
      constexpr int CPW = HD / 2;  // columns per warp
      const bool row_ok = key < s.T;
      const long long m = (long long)b * s.T + key;
      const int which = wq >> 1;  // 0: dK, 1: dV
      const int cbase = (wq & 1) * CPW;
      __nv_bfloat16* dst = dqkv + m * s.ld_qkv + (long long)(1 + which) * s.H * s.hdp + (long long)h * s.hdp;
      const uint32_t tsrc = (which == 0 ? tdK : tdV) + lane_off;
      const float f = which == 0 ? scale : 1.f;
#pragma unroll 1
      for (int c = cbase; c < cbase + CPW; c += 32) {
        float a[32];
        tmem_ld32(tsrc + c, a);
        if (row_ok) {
#pragma unroll
          for (int gg = 0; gg < 4; ++gg)
            reinterpret_cast<uint4*>(dst + c)[gg] =
                make_uint4(pack_bf16x2(a[8 * gg] * f, a[8 * gg + 1] * f), pack_bf16x2(a[8 * gg + 2] * f, a[8 * gg + 3] * f),
                           pack_bf16x2(a[8 * gg + 4] * f, a[8 * gg + 5] * f),
                           pack_bf16x2(a[8 * gg + 6] * f, a[8 * gg + 7] * f));
        }
      }
      // dK and dV have been read: the next item's products may overwrite them
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ====================================================================== backward: dQ
// Persistent like the dK/dV kernel: one CTA per SM walks (b, h, 128-query tile) items, heaviest
// tiles first, dealt in zigzag order; for each item it steps over 128-key blocks up to the
// diagonal one:
//   S = Q K^T and dP = dO V^T into TMEM (N = 128, full rate); sixteen elementwise warps write
//   dS = P (dP - delta) as bf16 into one of two TMEM buffers, from which dQ += dS K takes its
//   A operand.  S and dP are free again as soon as the elementwise warps have loaded them, so
//   the next block's S / dP products run while this block's dS is computed.
// TMEM: S [0,128), dP [128,256), dQ [256, 256+HD), dS [2] at 384 and 448.
// Shared memory: Q, dO, a 3-deep K ring (K is read by S and by dQ) and a 2-deep V ring; the
// rings run on across items, and the next item's Q and dO load once the current item's last
// S / dP products have read theirs.

template <int HD>
struct DqSmem {
  static constexpr int TILE = HD * 256;
  static constexpr int KS = 3, VS = 2;
  static constexpr int Q = 0;
  static constexpr int DO = Q + TILE;
  static constexpr int K0 = DO + TILE;        // [KS]
  static constexpr int V0 = K0 + KS * TILE;   // [VS]
  static constexpr int BAR = V0 + VS * TILE;
  static constexpr int BYTES = BAR + 256 + 1024;
};

// The key blocks of query tile qt: j0 .. qt (the last one is the diagonal block; j0 > 0 when the
// first query's window starts past key 0).
__device__ __forceinline__ int dq_first_block(const AttnShape& s, int qt) {
  return s.win >= 0 ? max(0, (qt * 128 - s.win) / 128) : 0;
}

template <int HD>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q128, const __grid_constant__ CUtensorMap tm_do128,
                       const __grid_constant__ CUtensorMap tm_kv128, const AttnShape s, const float* __restrict__ lse,
                       const float* __restrict__ delta, __nv_bfloat16* __restrict__ dqkv, float scale_log2,
                       float scale, DevCtl ctl) {
  using L = DqSmem<HD>;
  constexpr int KS = L::KS, VS = L::VS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;             // [KS]
  uint64_t* k_empty = k_full + KS;         // [KS]
  uint64_t* v_full = k_empty + KS;         // [VS]
  uint64_t* v_empty = v_full + VS;         // [VS]
  uint64_t* s_full = v_empty + VS;
  uint64_t* s_free = s_full + 1;
  uint64_t* ds_full = s_full + 2;          // [2]
  uint64_t* ds_empty = s_full + 4;         // [2]
  uint64_t* acc_full = s_full + 6;
  uint64_t* drain = s_full + 7;
  uint64_t* q_empty = s_full + 8;
  uint64_t* acc_empty = s_full + 9;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 10);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = (s.T + 127) / 128;
  const int BH = s.B * s.H;
  const int n_items = n_qt * BH;  // item w: query tile n_qt - 1 - w / BH (heaviest first), head w % BH
  constexpr int NCH = HD / 64;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < KS; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < VS; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, kBwdEw);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ds_full[i], kBwdEw);
      mbar_init(&ds_empty[i], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kBwdEw);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  pdl_wait();  // q, k, v (and dO, lse, delta) come from the kernels before this one
  const uint32_t tS = tbase;
  const uint32_t tdP = tbase + 128;
  const uint32_t tdQ = tbase + 256;
  const uint32_t tdS = tbase + 384;  // [2] x 64 columns

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA producer
    bool ok = true;
    int gj = 0;  // key blocks loaded, over all items
    int q_issued = -1, issued_k = -1, issued_v = -1;
    for (int r = 0; ok; ++r) {
      const int w = zigzag_item(r, blockIdx.x, gridDim.x);
      if (w >= n_items) break;
      const int qt = n_qt - 1 - w / BH, bh = w % BH;
      const int b = bh / s.H, h = bh % s.H;
      const int colq = h * s.hdp, cold = h * s.hdp;
      const int colk = s.H * s.hdp + h * s.hdp, colv = 2 * s.H * s.hdp + h * s.hdp;
      const int j0 = dq_first_block(s, qt);
      const int n_kv = qt + 1 - j0;
      // Q and dO of the previous item are read by its S / dP products until q_empty
      if (r > 0 && !mbar_wait(q_empty, (r - 1) & 1, ctl, abort_flag, 60)) { ok = false; break; }
      mbar_expect_tx(q_full, 2 * L::TILE);
      for (int c = 0; c < NCH; ++c) {
        tma_load_3d(sm + L::Q + c * 16384, &tm_q128, q_full, colq + 64 * c, qt * 128, b);
        tma_load_3d(sm + L::DO + c * 16384, &tm_do128, q_full, cold + 64 * c, qt * 128, b);
      }
      q_issued = r;
      for (int j = 0; j < n_kv && ok; ++j, ++gj) {
        const int ks = gj % KS;
        if (!mbar_wait(&k_empty[ks], ((gj / KS) & 1) ^ 1u, ctl, abort_flag, 60)) { ok = false; break; }
        mbar_expect_tx(&k_full[ks], L::TILE);
        for (int c = 0; c < NCH; ++c)
          tma_load_3d(sm + L::K0 + ks * L::TILE + c * 16384, &tm_kv128, &k_full[ks], colk + 64 * c, (j0 + j) * 128, b);
        issued_k = gj;
        const int vs = gj % VS;
        if (!mbar_wait(&v_empty[vs], ((gj / VS) & 1) ^ 1u, ctl, abort_flag, 61)) { ok = false; break; }
        mbar_expect_tx(&v_full[vs], L::TILE);
        for (int c = 0; c < NCH; ++c)
          tma_load_3d(sm + L::V0 + vs * L::TILE + c * 16384, &tm_kv128, &v_full[vs], colv + 64 * c, (j0 + j) * 128, b);
        issued_v = gj;
      }
    }
    if (!ok) {
      volatile int never = 0;
      if (q_issued >= 0) mbar_wait(q_full, q_issued & 1, ctl, &never, 62);
      for (int j = (issued_k >= KS ? issued_k - KS + 1 : 0); j <= issued_k && issued_k >= 0; ++j)
        mbar_wait(&k_full[j % KS], (j / KS) & 1, ctl, &never, 62);
      for (int j = (issued_v >= VS ? issued_v - VS + 1 : 0); j <= issued_v && issued_v >= 0; ++j)
        mbar_wait(&v_full[j % VS], (j / VS) & 1, ctl, &never, 62);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_s = idesc_bf16(128, 128, 0, 0);
    constexpr uint32_t idesc_d = idesc_bf16(128, HD, 0, 1);
    bool ok = true;
    bool issued = false;
    const uint64_t dQ = sdesc_sw128(smem_u32(sm + L::Q), 16, 1024);
    const uint64_t dD = sdesc_sw128(smem_u32(sm + L::DO), 16, 1024);
    const uint64_t dK0 = sdesc_sw128(smem_u32(sm + L::K0), 16, 1024);       // K-major, stage 0
    const uint64_t dKm0 = sdesc_sw128(smem_u32(sm + L::K0), 16384, 1024);   // MN-major, stage 0
    const uint64_t dV0 = sdesc_sw128(smem_u32(sm + L::V0), 16, 1024);
    // The block sequence over all items: S / dP of global block gj go out one step ahead of the
    // dQ product of block gj - 1, so that the next block's scores overlap this block's dS.
    int gj = 0;        // next block whose S / dP to issue
    int r_s = 0;       // item of block gj, and its block index within the item
    int j_s = 0;
    int n_s = -1;      // blocks of item r_s (-1: not yet looked up)
    int r_d = 0, j_d = 0, n_d = -1;  // the same for the next dQ product
    auto item_blocks = [&](int r) -> int {
      const int w = zigzag_item(r, blockIdx.x, gridDim.x);
      if (w >= n_items) return -1;
      const int qt = n_qt - 1 - w / BH;
      return qt + 1 - dq_first_block(s, qt);
    };
    n_s = item_blocks(0);
    n_d = n_s;
    int gd = 0;  // next block whose dQ product to issue
    while (ok && (n_s > 0 || n_d > 0)) {
      if (n_s > 0) {
        const int ks = gj % KS, vs = gj % VS;
        if (j_s == 0 && !mbar_wait(q_full, r_s & 1, ctl, abort_flag, 63)) { ok = false; break; }
        if (!mbar_wait(&k_full[ks], (gj / KS) & 1, ctl, abort_flag, 64)) { ok = false; break; }
        if (!mbar_wait(&v_full[vs], (gj / VS) & 1, ctl, abort_flag, 64)) { ok = false; break; }
        // S / dP are free once the elementwise warps have loaded the previous block's
        if (gj > 0 && !mbar_wait(s_free, (gj - 1) & 1, ctl, abort_flag, 65)) { ok = false; break; }
        tc_fence_after();
        const uint64_t dK = sdesc_add(dK0, ks * L::TILE);
        const uint64_t dV = sdesc_add(dV0, vs * L::TILE);
#pragma unroll
        for (int gq = 0; gq < HD / 64; ++gq) {
          uint32_t dd[8];
          uint64_t aa[8], bb[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t off = gq * 16384 + i * 32;
            dd[2 * i] = tS;
            dd[2 * i + 1] = tdP;
            aa[2 * i] = sdesc_add(dQ, off);
            aa[2 * i + 1] = sdesc_add(dD, off);
            bb[2 * i] = sdesc_add(dK, off);
            bb[2 * i + 1] = sdesc_add(dV, off);
          }
          umma8_ss(dd, aa, bb, idesc_s, gq == 0 ? 0xfcu : 0xffu);
        }
        umma_commit(s_full);
        umma_commit(&v_empty[vs]);
        if (j_s == n_s - 1) umma_commit(q_empty);  // the item's Q and dO are no longer read
        issued = true;
        ++gj;
        if (++j_s == n_s) {
          ++r_s;
          j_s = 0;
          n_s = item_blocks(r_s);
        }
      }
      if (gd < gj - 1 || (n_s <= 0 && gd < gj)) {
        // dQ += dS K of block gd, issued after the S / dP products of block gd + 1 (if any)
        const int bb = gd & 1;
        if (!mbar_wait(&ds_full[bb], (gd >> 1) & 1, ctl, abort_flag, 66)) { ok = false; break; }
        // the item's first dQ product overwrites the previous item's dQ: read out by then
        if (j_d == 0 && r_d > 0 && !mbar_wait(acc_empty, (r_d - 1) & 1, ctl, abort_flag, 68)) { ok = false; break; }
        tc_fence_after();
        const uint64_t dKm = sdesc_add(dKm0, (gd % KS) * L::TILE);
        const uint32_t tA = tdS + 64 * bb;
        uint32_t dd[8], aa[8];
        uint64_t bd[8];
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // 16 keys each
          dd[kk] = tdQ;
          aa[kk] = tA + 8 * kk;
          bd[kk] = sdesc_add(dKm, kk * 2048);
        }
        umma8_ts(dd, aa, bd, idesc_d, j_d == 0 ? 0xfeu : 0xffu);
        umma_commit(&ds_empty[bb]);
        umma_commit(&k_empty[gd % KS]);
        issued = true;
        ++gd;
        if (++j_d == n_d) {
          umma_commit(acc_full);
          ++r_d;
          j_d = 0;
          n_d = item_blocks(r_d);
        }
      }
    }
    if (!ok && issued) {
      volatile int never = 0;
      umma_commit(drain);
      mbar_wait(drain, 0, ctl, &never, 67);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------ elementwise warps
    const int ew = warp - 2;
    const int quad = warp & 3;  // TMEM lane quadrant: queries 32 quad .. 32 quad + 31
    const int cg = ew >> 2;     // key columns 32 cg .. 32 cg + 31 of each block
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    bool ok = true;
    int gj = 0;
    for (int r = 0; ok; ++r) {
      const int w = zigzag_item(r, blockIdx.x, gridDim.x);
      if (w >= n_items) break;
      const int qt = n_qt - 1 - w / BH, bh = w % BH;
      const int b = bh / s.H, h = bh % s.H;
      const int q0 = qt * 128;
      const int j0 = dq_first_block(s, qt);
      const int n_kv = qt + 1 - j0;
      const int qi = q0 + quad * 32 + lane;
      const bool row_ok = qi < s.T;
      const float lse2 = row_ok ? lse[(long long)bh * s.T + qi] * kLog2e : 0.f;
      const float dl = row_ok ? delta[(long long)bh * s.T + qi] : 0.f;
      for (int j = 0; j < n_kv; ++j, ++gj) {
        if (!mbar_wait(s_full, gj & 1, ctl, abort_flag, 68)) { ok = false; break; }
        tc_fence_after();
        uint32_t rs[32], rd[32];
        tmem_ld32_nowait(tS + lane_off + 32 * cg, rs);
        tmem_ld32_nowait(tdP + lane_off + 32 * cg, rd);
        tmem_wait_ld();
        tmem_fence_regs<32>(rs);
        tmem_fence_regs<32>(rd);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
        const int bb = gj & 1;
        if (!mbar_wait(&ds_empty[bb], ((gj >> 1) & 1) ^ 1u, ctl, abort_flag, 69)) { ok = false; break; }
        const int kb = (j0 + j) * 128 + 32 * cg;
        uint32_t dw[16];
        if ((kb + 31 > q0) || (kb + 32 > s.T) || !row_ok || (s.win >= 0 && kb < q0 + 127 - s.win)) {
          // diagonal block, ragged end, rows past T or the window's lower edge: mask
#pragma unroll
          for (int e2 = 0; e2 < 16; ++e2) {
            float d2[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              const int e = 2 * e2 + k;
              const int key = kb + e;
              float pv = ex2_approx(fmaf(__uint_as_float(rs[e]), scale_log2, -lse2));
              if (!row_ok || key > qi || key >= s.T || (s.win >= 0 && key < qi - s.win)) pv = 0.f;
              d2[k] = pv * (__uint_as_float(rd[e]) - dl);
            }
            dw[e2] = pack_bf16x2(d2[0], d2[1]);
          }
        } else {
#pragma unroll
          for (int e2 = 0; e2 < 16; ++e2) {
            const float p0 = ex2_approx(fmaf(__uint_as_float(rs[2 * e2]), scale_log2, -lse2));
            const float p1 = ex2_approx(fmaf(__uint_as_float(rs[2 * e2 + 1]), scale_log2, -lse2));
            dw[e2] = pack_bf16x2(p0 * (__uint_as_float(rd[2 * e2]) - dl), p1 * (__uint_as_float(rd[2 * e2 + 1]) - dl));
          }
        }
        tmem_st16(tdS + 64 * bb + lane_off + 16 * cg, dw);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ds_full[bb]);
      }
      if (!ok) break;
      if (!mbar_wait(acc_full, r & 1, ctl, abort_flag, 70)) { ok = false; break; }
      tc_fence_after();
      // the four warps of a quadrant split dQ's columns
      constexpr int CPW = HD / 4;
      __nv_bfloat16* dq = dqkv + ((long long)b * s.T + qi) * s.ld_qkv + (long long)h * s.hdp + cg * CPW;
      if (CPW == 32) {
        float a[32];
        tmem_ld32(tdQ + lane_off + cg * CPW, a);
        if (row_ok) {
#pragma unroll
          for (int g = 0; g < 4; ++g)
            reinterpret_cast<uint4*>(dq)[g] = make_uint4(
                pack_bf16x2(a[8 * g] * scale, a[8 * g + 1] * scale), pack_bf16x2(a[8 * g + 2] * scale, a[8 * g + 3] * scale),
                pack_bf16x2(a[8 * g + 4] * scale, a[8 * g + 5] * scale),
                pack_bf16x2(a[8 * g + 6] * scale, a[8 * g + 7] * scale));
        }
      } else {
        uint32_t a[16];
        tmem_ld16_nowait(tdQ + lane_off + cg * CPW, a);
        tmem_wait_ld();
        tmem_fence_regs<16>(a);
        if (row_ok) {
#pragma unroll
          for (int g = 0; g < 2; ++g)
            reinterpret_cast<uint4*>(dq)[g] = make_uint4(
                pack_bf16x2(__uint_as_float(a[8 * g]) * scale, __uint_as_float(a[8 * g + 1]) * scale),
                pack_bf16x2(__uint_as_float(a[8 * g + 2]) * scale, __uint_as_float(a[8 * g + 3]) * scale),
                pack_bf16x2(__uint_as_float(a[8 * g + 4]) * scale, __uint_as_float(a[8 * g + 5]) * scale),
                pack_bf16x2(__uint_as_float(a[8 * g + 6]) * scale, __uint_as_float(a[8 * g + 7]) * scale));
        }
      }
      // dQ has been read: the next item's products may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ====================================================================== launchers

double attn_pairs(int T, int win) {
  const double t = T;
  if (win < 0 || win >= T - 1) return t * (t + 1) / 2;
  const double w = win;
  return w * (w + 1) / 2 + (t - w) * (w + 1);  // rows i < win see i + 1 keys, the rest win + 1
}

template <int HD>
static int attn_fwd_launch(const CUtensorMap& tm, const AttnShape& s, __nv_bfloat16* o, long long ldo, float* lse,
                           float scale_log2, float* amax, cudaStream_t st) {
  using L = FwdSmem<HD>;
  GPTK_CUDA(cudaFuncSetAttribute(attn_fwd_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES));
  // setmaxnreg.inc waits until the registers it asks for are free in the block's own allocation:
  // launch only with the allocation the split was made for
  static const int regs = [] {
    cudaFuncAttributes fa;
    return cudaFuncGetAttributes(&fa, attn_fwd_kernel<HD>) == cudaSuccess ? fa.numRegs : 0;
  }();
  if (regs * kFwdThreads < 128 * kFwdRegsProducer + 256 * kFwdRegsSoftmax)
    return set_error(ST_CUDA, "attention forward: built with fewer registers per thread than its warpgroup split");
  // (b, h) fastest, so the heaviest causal pairs of every head start first
  dim3 grid(s.B * s.H, (s.T + 255) / 256);
  const double causal = (double)s.B * s.H * attn_pairs(s.T, s.win);
  Prof prof(PK_ATTN_FWD, 4.0 * s.hd * causal, (double)s.B * s.T * s.H * s.hd * 2 * 4, st);
  GPTK_CUDA(launch_pdl(attn_fwd_kernel<HD>, grid, dim3(kFwdThreads), L::BYTES, st, tm, s, o, ldo, lse, scale_log2,
                       reinterpret_cast<unsigned int*>(amax), device_ctl()));
  GPTK_CUDA(cudaGetLastError());
  return ST_OK;
}

template <int HD>
static int attn_fwd_t(const __nv_bfloat16* qkv, const AttnShape& s, __nv_bfloat16* o, long long ldo, float* lse,
                      float* amax, cudaStream_t st) {
  CUtensorMap tm;
  GPTK_TRY(make_tmap_3d(&tm, qkv, 3ull * s.H * s.hdp, s.T, s.B, s.ld_qkv, (uint64_t)s.T * s.ld_qkv, 64, 128, 1));
  return attn_fwd_launch<HD>(tm, s, o, ldo, lse, kLog2e / sqrtf((float)s.hd), amax, st);
}

int launch_attn_fwd(const __nv_bfloat16* qkv_pad, const AttnShape& s, __nv_bfloat16* o, long long ldo, float* lse,
                    cudaStream_t st, float* amax) {
  if (s.B < 1 || s.T < 1 || s.H < 1) return set_error(ST_INVALID_ARG, "attention: empty shape");
  if (s.win < -1) return set_error(ST_INVALID_ARG, "attention: window must be >= 0 (or -1 for none)");
  if (s.B * s.H > 65535) return set_error(ST_UNSUPPORTED, "attention: B*H above 65535");
  if (s.hdp == 64) return attn_fwd_t<64>(qkv_pad, s, o, ldo, lse, amax, st);
  if (s.hdp == 128) return attn_fwd_t<128>(qkv_pad, s, o, ldo, lse, amax, st);
  return set_error(ST_UNSUPPORTED, "attention: padded head dim must be 64 or 128");
}

template <int HD>
static int attn_bwd_t(const __nv_bfloat16* qkv, const __nv_bfloat16* dop, const float* lse, const float* delta,
                      const AttnShape& s, __nv_bfloat16* dqkv, cudaStream_t st) {
  const uint64_t ldd = (uint64_t)s.H * s.hdp;
  // 128-row boxes of one 64-column chunk of q, k, v (the padded q|k|v buffer) and of dO
  CUtensorMap qkv128, do128;
  GPTK_TRY(make_tmap_3d(&qkv128, qkv, 3ull * s.H * s.hdp, s.T, s.B, s.ld_qkv, (uint64_t)s.T * s.ld_qkv, 64, 128, 1));
  GPTK_TRY(make_tmap_3d(&do128, dop, ldd, s.T, s.B, ldd, (uint64_t)s.T * ldd, 64, 128, 1));
  const float scale = 1.f / sqrtf((float)s.hd);
  const float scale_log2 = kLog2e * scale;
  const DevCtl ctl = device_ctl();
  const double causal = (double)s.B * s.H * attn_pairs(s.T, s.win);
  {
    using L = DkvSmem<HD>;
    static_assert(L::BYTES <= 232448, "dK/dV shared memory above the per-block limit");
    GPTK_CUDA(cudaFuncSetAttribute(attn_bwd_dkv_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES));
    // persistent: one CTA per SM over the (key tile, head) items
    const long long items = (long long)((s.T + 127) / 128) * s.B * s.H;
    dim3 grid((unsigned)std::min<long long>(items, num_sms()));
    Prof prof(PK_ATTN_BWD_DKV, 8.0 * s.hd * causal, (double)s.B * s.T * s.H * s.hd * 2 * 6, st);
    GPTK_CUDA(launch_pdl(attn_bwd_dkv_kernel<HD>, grid, dim3(kBwdThreads), L::BYTES, st, qkv128, qkv128, do128, s, lse,
                         delta, dqkv, scale_log2, scale, ctl));
    GPTK_CUDA(cudaGetLastError());
  }
  {
    using L = DqSmem<HD>;
    static_assert(L::BYTES <= 232448, "dQ shared memory above the per-block limit");
    GPTK_CUDA(cudaFuncSetAttribute(attn_bwd_dq_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES));
    const long long items = (long long)((s.T + 127) / 128) * s.B * s.H;
    dim3 grid((unsigned)std::min<long long>(items, num_sms()));
    Prof prof(PK_ATTN_BWD_DQ, 6.0 * s.hd * causal, (double)s.B * s.T * s.H * s.hd * 2 * 5, st);
    GPTK_CUDA(launch_pdl(attn_bwd_dq_kernel<HD>, grid, dim3(kBwdThreads), L::BYTES, st, qkv128, do128, qkv128, s, lse,
                         delta, dqkv, scale_log2, scale, ctl));
    GPTK_CUDA(cudaGetLastError());
  }
  return ST_OK;
}

int launch_attn_bwd(const __nv_bfloat16* qkv_pad, const __nv_bfloat16* do_pad, const float* lse,
                    const float* delta, const AttnShape& s, __nv_bfloat16* dqkv_pad, cudaStream_t st) {
  if (s.B < 1 || s.T < 1 || s.H < 1) return set_error(ST_INVALID_ARG, "attention: empty shape");
  if (s.win < -1) return set_error(ST_INVALID_ARG, "attention: window must be >= 0 (or -1 for none)");
  if (s.B * s.H > 65535) return set_error(ST_UNSUPPORTED, "attention: B*H above 65535");
  if (s.hdp == 64) return attn_bwd_t<64>(qkv_pad, do_pad, lse, delta, s, dqkv_pad, st);
  if (s.hdp == 128) return attn_bwd_t<128>(qkv_pad, do_pad, lse, delta, s, dqkv_pad, st);
  return set_error(ST_UNSUPPORTED, "attention: padded head dim must be 64 or 128");
}

}  // namespace gptk
