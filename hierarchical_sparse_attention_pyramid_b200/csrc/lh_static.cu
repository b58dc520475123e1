// lh_score_topk_static: the stage-2 selection without any caller-provided or
// library-allocated workspace.
//
// lh_score_topk keeps its max-pooled score pyramid in the ws buffer that the
// caller allocates.  Some callers cannot allocate device memory at the point
// where they run the selection: a host application whose allocator owns every
// device buffer and hands out only the tensors of a call, an inference or
// training runtime that forbids allocations once its memory plan is fixed, or
// a plugin that is only given its inputs and outputs.  For them this entry
// point keeps the score pyramid in one file-scope device array of fixed size
// that the library carries from load to exit, and calls no allocator.
#include <cuda.h>
#include <mutex>

#include "lh_common.cuh"

namespace lh {
namespace {

// Largest scratch the static array holds: 16 MiB.  A call needs the score
// pyramid, B*H times the entries of levels >= 1 times 4 bytes, plus (direct
// selection only) the level-0 scores, B*H*N*4 bytes, after it: lh_plan's
// topk_ws_bytes minus the error word.  The 512K-token, 16-head layer needs
// 11.1 MB (45 MB with direct selection, which is refused); the 1M-token,
// 8-head layer 11.2 MB.
constexpr size_t kStaticScratchBytes = size_t(16) << 20;

// Held by every GPU that loads the library until the process exits.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 128;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

// The current context, read through the runtime's driver entry point (no
// link against libcuda).  A cudaDeviceReset replaces the device's primary
// context, which reloads the module and can move the array.
CUcontext current_context() {
  using Fn = CUresult (*)(CUcontext*);
  static Fn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<Fn>(p);
  }
  CUcontext c = nullptr;
  if (fn) fn(&c);
  return c;
}

// Device address of the array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress (with that device current) and cached per device,
// keyed by the context it was looked up in: a call in a new context (after a
// cudaDeviceReset) looks it up again.
cudaError_t scratch_on_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const CUcontext ctx = current_context();  // NULL before the runtime made one current
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev] || !ctx || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);  // makes the primary context current if none is
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = current_context();
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace lh

extern "C" lh_status lh_score_topk_static(const lh_config* cfg, const float* norms, int32_t* sel,
                                           lh_stream_t stream) {
  using namespace lh;
  lh_plan_info info;
  Dims D;
  lh_status s = make_dims(cfg, &info, &D);
  if (s != LH_OK) return s;
  if (D.L == 1) return LH_OK;
  if (!norms || !sel || (reinterpret_cast<uintptr_t>(norms) & 15u) || (reinterpret_cast<uintptr_t>(sel) & 15u)) {
    set_error_message("lh_score_topk_static: norms or sel is NULL or not 16-byte aligned");
    return LH_ERR_INVALID_ARG;
  }
  // the score pyramid, and (direct selection) the level-0 scores after it
  const size_t need = info.topk_ws_bytes - LH_ERR_WORD_BYTES;
  if (need > kStaticScratchBytes) {
    set_error_message("lh_score_topk_static: the score pyramid needs %zu bytes but the static scratch holds %zu; "
                      "use lh_score_topk with a caller-provided ws",
                      need, kStaticScratchBytes);
    return LH_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  cudaError_t e = scratch_on_current_device(&scratch);
  if (e != cudaSuccess) {
    set_error_message("lh_score_topk_static: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    return LH_ERR_CUDA;
  }
  // every entry of the pyramid is written before it is read, so nothing in
  // the array has to start at zero.  There is no error word: the one
  // device-side check of the selection (a nested chunk larger than its
  // staging buffer) is kept unreachable by lh_plan's limits.
  e = launch_score_topk(D, norms, static_cast<float*>(scratch), sel, nullptr, (cudaStream_t)stream);
  if (e != cudaSuccess) {
    set_error_message("lh_score_topk_static: %s", cudaGetErrorString(e));
    return LH_ERR_CUDA;
  }
  return LH_OK;
}
