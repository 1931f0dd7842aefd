// lm_head + cross-entropy forward for callers that cannot allocate device memory.
//
// gpt_op_lmhead_ce_fwd asks its caller for scratch (the per-row partial
// logsumexp of every vocab tile, plus each row's target logit).  Some callers
// cannot hand out device memory on this path: a serving or training loop whose
// device memory is entirely reserved up front by its own pool, where a
// cudaMalloc would fail or fragment that pool, or code that cannot afford the
// device-wide synchronisation a cudaMalloc / cudaFree may bring in the middle
// of a step.  This variant keeps that scratch in a fixed file-scope device
// array instead, so the call allocates nothing.
//
// The array is kNoAllocScratchBytes (16 MiB) on every GPU that loads the
// library, held until the process exits.  Host code cannot pass the array's
// name to a kernel (on the host it is only a stand-in symbol), so the first
// call on each device looks up its device address with cudaGetSymbolAddress,
// with that device current, and caches it once the lookup has succeeded; make
// that first call before any stream capture.  All calls share the one array and
// it keeps the last call's contents: the target-logit slots are cleared at the
// start of every call (a row whose target lies outside [0, V) gets a NaN loss
// and a device status report, never a stale value), and calls that overlap on
// the GPU (different streams, no ordering between them) race on the array.
#include <mutex>
#include <string>

#include "gemm.cuh"
#include "gpt_ops.h"
#include "host.cuh"
#include "kernels.cuh"

namespace gptk {

static constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;

static __device__ __align__(256) unsigned char g_ce_scratch[kNoAllocScratchBytes];

static void* g_ce_scratch_addr[64];  // non-null once found on that device
static std::mutex g_ce_scratch_mu;

// Device address of g_ce_scratch on the current device.  Only a successful lookup is kept: a
// failed one (an error left pending by an earlier launch, or a first call made while a stream
// is being captured) is retried by the next call instead of failing every later call.
static int ce_scratch_address(void** out) {
  int dev = 0;
  GPTK_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return set_error(ST_UNSUPPORTED, "lmhead_ce_noalloc: device index above 63");
  std::lock_guard<std::mutex> lock(g_ce_scratch_mu);
  if (g_ce_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_ce_scratch);
    if (e != cudaSuccess || p == nullptr)
      return set_error(ST_CUDA, std::string("lmhead_ce_noalloc: cudaGetSymbolAddress failed: ") +
                                    cudaGetErrorString(e));
    g_ce_scratch_addr[dev] = p;
  }
  *out = g_ce_scratch_addr[dev];
  return ST_OK;
}

}  // namespace gptk

using namespace gptk;

extern "C" {

GPT_API size_t gpt_op_lmhead_ce_noalloc_max_scratch_bytes(void) { return kNoAllocScratchBytes; }

GPT_API int gpt_op_lmhead_ce_fwd_noalloc(const void* x, const void* w, const int32_t* targets, int M, int D, int V,
                                         float* ell, float* lse, void* stream) {
  set_error(ST_OK, "");
  if (!x || !w || !targets || !ell || !lse) return set_error(ST_INVALID_ARG, "lmhead_ce_noalloc: null pointer");
  if (M < 1 || D < 1 || V < 1) return set_error(ST_INVALID_ARG, "lmhead_ce_noalloc: M, D, V must be >= 1");
  if (D % 8) return set_error(ST_UNSUPPORTED, "lmhead_ce_noalloc: D must be a multiple of 8");
  const size_t ntn = (size_t)(V + 255) / 256;
  const size_t part_bytes = ((size_t)M * ntn * 8 + 255) / 256 * 256;
  const size_t need = part_bytes + ((size_t)M * 4 + 255) / 256 * 256;
  if (need > kNoAllocScratchBytes)
    return set_error(ST_INVALID_ARG, "lmhead_ce_noalloc: M=" + std::to_string(M) + ", V=" + std::to_string(V) +
                                         " needs " + std::to_string(need) + " bytes of scratch, above the fixed " +
                                         std::to_string(kNoAllocScratchBytes) +
                                         "; split the rows or use gpt_op_lmhead_ce_fwd");
  void* base = nullptr;
  GPTK_TRY(ce_scratch_address(&base));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float2* part = static_cast<float2*>(base);
  float* zy = reinterpret_cast<float*>(static_cast<char*>(base) + part_bytes);
  // the array keeps the previous call's values: clear the target-logit slots
  GPTK_CUDA(cudaMemsetAsync(zy, 0, (size_t)M * 4, st));
  GemmParams p = {};
  p.M = M;
  p.N = V;
  p.K = D;
  p.hd = p.hdp = 1;
  p.targets = targets;
  p.ce_part = part;
  p.ce_zy = zy;
  GPTK_TRY(run_gemm(EPI_CE_FWD, 256, Operand{x, D, 0}, Operand{w, D, 0}, p, st));
  return launch_ce_combine(part, (int)ntn, zy, targets, V, M, ell, lse, st);
}

}  // extern "C"
