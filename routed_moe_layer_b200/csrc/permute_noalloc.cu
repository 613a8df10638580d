// moe_permute_noalloc: the token -> expert permutation without a caller
// workspace.  The kernels are the ones moe_permute launches; their scratch
// (status word, per-block expert histograms, tile prefix) lives in a
// file-scope device array of fixed size instead of caller memory, so the
// call allocates nothing.
#include <mutex>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "routed_moe.h"

namespace {

constexpr int kMaxBlocks = (MOE_NOALLOC_MAX_T + rmoe::PERMUTE_TOK - 1) / rmoe::PERMUTE_TOK;
constexpr int kMaxExperts = 128;  // the limit moe_check_config enforces
constexpr size_t kStatusOff = 0;
constexpr size_t kHistOff = 256;
constexpr size_t kTilesOff = kHistOff + (size_t)kMaxBlocks * kMaxExperts * sizeof(int);
constexpr size_t kScratchBytes = kTilesOff + (kMaxExperts + 1) * sizeof(int);

}  // namespace

// One copy per device that loads the library, held until the process exits
// (about 129 KiB).  In host code this name is only a handle for the runtime:
// the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_permute_scratch[kScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // id of the context the address belongs to

PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;

// Unique id of the calling thread's current context, 0 when there is none
// (or the driver cannot tell).
unsigned long long current_context_id() {
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!g_ctx_current || !g_ctx_id || g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (g_ctx_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_permute_scratch on the current device, looked up once
// per device (with that device current) and cached with the id of the
// context it belongs to.  A device reset destroys that context and the next
// call makes a new one: the id then differs and the address is looked up again.
int32_t scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  const unsigned long long ctx = current_context_id();
  if (g_scratch_ptr[dev] == nullptr || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr)
      return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = p;
    // the lookup made the device's context current if it was not yet
    g_scratch_ctx[dev] = ctx != 0 ? ctx : current_context_id();
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" int32_t moe_permute_noalloc(const int32_t* topk_ids, const float* topk_w,
                                       const void* x, const moe_cfg_t* cfg,
                                       int32_t* expert_offsets, int32_t* row_of, int32_t* tok_of,
                                       float* w_of, void* xp, void* stream) {
  const int32_t st = moe_check_config(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T == 0) return MOE_OK;
  if (cfg->T > MOE_NOALLOC_MAX_T) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!topk_ids || !expert_offsets || !row_of || !tok_of) return MOE_ERR_INVALID_ARG;
  if (xp && !x) return MOE_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const int32_t sst = scratch_address(&scratch);
  if (sst != MOE_OK) return sst;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(scratch);
  int* status = reinterpret_cast<int*>(base + kStatusOff);
  // the histograms and tile prefix are fully rewritten by every call; only the
  // status word must start at zero
  if (rmoe::launch_status_reset(status, s) != cudaSuccess) return MOE_ERR_CUDA;
  rmoe::PermuteOut o;
  o.status = status;
  o.blk_hist = reinterpret_cast<int*>(base + kHistOff);
  o.expert_offsets = expert_offsets;
  o.mtile_start = reinterpret_cast<int*>(base + kTilesOff);
  o.row_of = row_of;
  o.tok_of = tok_of;
  o.w_of = w_of;
  o.xp = xp;
  return rmoe::launch_permute(topk_ids, topk_w, x, cfg->T, cfg->H, cfg->E, cfg->top_k, o, s) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}
