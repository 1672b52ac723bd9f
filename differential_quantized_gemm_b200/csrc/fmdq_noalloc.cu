// dstar_fmdq_linear_noalloc: the FMDQ differential linear for callers that
// cannot allocate device memory.  Its scratch is a static device array of this
// file instead of a caller-owned workspace; the computation is exactly that of
// dstar_fmdq_linear, which it calls with the array as the workspace.
//
// In host code the name of a __device__ array only stands for it: the address
// a kernel needs comes from cudaGetSymbolAddress, looked up on every call with
// the caller's device current (cheap once the module is loaded).  A device
// reset or a new primary context loads the module again, possibly at another
// address and with stale contents, so the one-time clearing of the status word
// is keyed to the context's unique ID, never to the device number.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "fmdq_internal.h"

// Scratch of dstar_fmdq_linear_noalloc: one copy on every device that loads
// this library, held until the process exits.  256-byte alignment is what the
// workspace layout asks of its base.
static __device__ __align__(256) uint8_t g_noalloc_scratch[DSTAR_NOALLOC_SCRATCH_BYTES];

namespace fmdq {
namespace {

// IDs of the contexts whose copy of the array has had its status word cleared
// (a small ring; re-clearing after an eviction is harmless).
constexpr int kMaxContexts = 64;
std::mutex g_scratch_mu;
unsigned long long g_cleared[kMaxContexts] = {};
int g_ncleared = 0, g_next = 0;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique ID (for the life of the process) of the calling thread's current context.
int current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!get_current || !get_id) return report_error(DSTAR_ERR_CUDA, "cuCtxGetCurrent/cuCtxGetId are not available");
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return report_error(DSTAR_ERR_CUDA, "no current CUDA context");
  if (get_id(ctx, id) != CUDA_SUCCESS) return report_error(DSTAR_ERR_CUDA, "cuCtxGetId failed");
  return DSTAR_OK;
}

// Device address of the scratch in the current context.  The first call in a
// context enqueues the clearing of the status word on `stream` (the only part
// of the workspace that must start at zero).
int scratch_address(void** out, cudaStream_t stream) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // makes the primary context current if needed
  if (e != cudaSuccess) return report_cuda_error(e, "cudaGetSymbolAddress of the static scratch");
  unsigned long long id = 0;
  int r = current_context_id(&id);
  if (r != DSTAR_OK) return r;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  bool cleared = false;
  for (int i = 0; i < g_ncleared && !cleared; ++i) cleared = g_cleared[i] == id;
  if (!cleared) {
    e = cudaMemsetAsync(p, 0, 256, stream);
    if (e != cudaSuccess) return report_cuda_error(e, "clearing the static scratch's status word");
    g_cleared[g_next] = id;
    g_next = (g_next + 1) % kMaxContexts;
    if (g_ncleared < kMaxContexts) ++g_ncleared;
  }
  *out = p;
  return DSTAR_OK;
}

}  // namespace
}  // namespace fmdq

using namespace fmdq;

extern "C" int dstar_fmdq_linear_noalloc(const dstar_mat* x_t, dstar_mat* x_prev, dstar_mat* y_prev,
                                         const dstar_mat* w_q, const float* w_scale, float base_scale,
                                         const dstar_tile_cfg* tile_cfg, dstar_mat* y_out, uint32_t* status_out,
                                         void* stream) {
  if (!tile_cfg) return report_error(DSTAR_ERR_INVALID_ARG, "tile_cfg is NULL");
  if (tile_cfg->workspace || tile_cfg->workspace_bytes)
    return report_error(DSTAR_ERR_INVALID_ARG,
                        "dstar_fmdq_linear_noalloc uses its own static scratch: tile_cfg->workspace must be NULL "
                        "and workspace_bytes 0");
  if (!x_t) return report_error(DSTAR_ERR_INVALID_ARG, "x_t is NULL");
  if (status_out && (reinterpret_cast<uintptr_t>(status_out) & 3u))
    return report_error(DSTAR_ERR_INVALID_ARG, "status_out must be 4-byte aligned");
  const int64_t M = x_t->rows, K = x_t->cols;
  if (M < 0 || M % kTile != 0 || K <= 0 || K % 32 != 0 || K > DSTAR_K_MAX)
    return report_error(DSTAR_ERR_INVALID_ARG,
                        "x_t must have M % 16 == 0 rows and 0 < K <= 8192 columns with K % 32 == 0");
  const size_t need = ws_layout(M, K).total;
  if (need > (size_t)DSTAR_NOALLOC_SCRATCH_BYTES) {
    char msg[256];
    snprintf(msg, sizeof msg,
             "M=%lld, K=%lld needs %zu bytes of scratch, more than the %zu-byte static scratch of "
             "dstar_fmdq_linear_noalloc; split the tokens or use dstar_fmdq_linear with a workspace",
             (long long)M, (long long)K, need, (size_t)DSTAR_NOALLOC_SCRATCH_BYTES);
    return report_error(DSTAR_ERR_WORKSPACE, msg);
  }

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  int r = scratch_address(&scratch, s);
  if (r != DSTAR_OK) return r;
  dstar_tile_cfg cfg = *tile_cfg;
  cfg.workspace = scratch;
  cfg.workspace_bytes = DSTAR_NOALLOC_SCRATCH_BYTES;
  r = dstar_fmdq_linear(x_t, x_prev, y_prev, w_q, w_scale, base_scale, &cfg, y_out, stream);
  if (r != DSTAR_OK) {
    // a launch failed part-way: leave the status word clear for the next call
    if (r == DSTAR_ERR_CUDA) (void)cudaMemsetAsync(scratch, 0, sizeof(uint32_t), s);
    return r;
  }
  cudaError_t e = cudaSuccess;
  if (status_out)
    e = cudaMemcpyAsync(status_out, scratch, sizeof(uint32_t), cudaMemcpyDefault, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(scratch, 0, sizeof(uint32_t), s);
  if (e != cudaSuccess) return report_cuda_error(e, "passing on the status word");
  return DSTAR_OK;
}
