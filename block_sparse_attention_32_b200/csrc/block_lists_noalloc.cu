// Allocation-free variant of msa_build_block_query_lists.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the point
// where they build the block->query lists: a plugin running inside a serving
// process whose host owns all device memory through its own pool, or a
// latency-critical loop that must not allocate.  For them this entry point
// takes no workspace: the inversion's scratch lives in a file-scope device
// array of fixed size that every GPU loading the library keeps until the
// process exits.  The arithmetic is exactly that of the workspace version (the
// same kernels are launched, only the scratch pointer differs).
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"

namespace msa {
cudaError_t launch_block_lists(const int32_t* sel, int64_t bgcount, int64_t n_q, int64_t q_pos0,
                               int64_t nblk, int64_t window, int32_t* offsets, int32_t* entries,
                               int32_t* entry_pos, int64_t cap, void* ws, int32_t* err,
                               cudaStream_t st);
msa_status validate_dims(const msa_dims* d);
}  // namespace msa

// The scratch.  In host code this name is only a host-side stand-in for the
// device symbol: its device address must be obtained with
// cudaGetSymbolAddress on each device before it is handed to a kernel.  The
// array belongs to this file's device module, which no kernel launch loads:
// under CUDA's default lazy module loading the 32 MiB are committed on a
// device by the first cudaGetSymbolAddress there, i.e. by the first call of
// the entry point on that device (under CUDA_MODULE_LOADING=EAGER, when the
// library's context is created).
static __device__ __align__(256) unsigned char g_block_lists_scratch[MSA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
// per device: the context the address was looked up in, and the address
void* g_scratch_ctx[kMaxDevices] = {};
void* g_scratch_ptr[kMaxDevices] = {};

// cuCtxGetCurrent through the runtime's driver entry point (no libcuda link)
PFN_cuCtxGetCurrent_v4000 ctx_current_fn() {
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  });
  return fn;
}

// Device address of the scratch on the current device.  It is looked up with
// that device current the first time the entry point runs in a context, and
// again whenever the device's current context has changed since (after a
// cudaDeviceReset the module is loaded anew and the array may move), so a
// stale address is never handed to a kernel.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  auto get_ctx = ctx_current_fn();
  if (get_ctx == nullptr) return cudaErrorNotSupported;
  // null while this thread has not used the runtime on the device yet
  CUcontext c = nullptr;
  if (get_ctx(&c) != CUDA_SUCCESS) return cudaErrorContextIsDestroyed;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (c == nullptr || g_scratch_ptr[dev] == nullptr || g_scratch_ctx[dev] != (void*)c) {
    void* p = nullptr;
    // also makes the device's primary context current on this thread
    e = cudaGetSymbolAddress(&p, g_block_lists_scratch);
    if (e != cudaSuccess) return e;
    if (p == nullptr) return cudaErrorInvalidSymbol;
    if (get_ctx(&c) != CUDA_SUCCESS || c == nullptr) return cudaErrorContextIsDestroyed;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = (void*)c;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" msa_status msa_build_block_query_lists_noalloc(const msa_dims* d, const int32_t* sel,
                                                          int32_t* blk_offsets, int32_t* entries,
                                                          int32_t* entry_pos, int32_t* dev_err,
                                                          void* stream) {
  // the workspace version's checks, with its status codes
  msa_status s = msa::validate_dims(d);
  if (s != MSA_OK) return s;
  if (sel == nullptr || blk_offsets == nullptr || entries == nullptr || entry_pos == nullptr)
    return MSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(sel) & 15u) != 0) return MSA_ERR_ALIGNMENT;
  const size_t need = msa_block_query_lists_workspace(d);
  if (need > (size_t)MSA_NOALLOC_SCRATCH_BYTES) return MSA_ERR_SCRATCH_LIMIT;
  const int64_t total = msa_num_entries(d);
  if (total >= (int64_t(1) << 31)) return MSA_ERR_UNSUPPORTED;
  void* ws = nullptr;
  if (scratch_address(&ws) != cudaSuccess) {
    // leave no error behind for the next call that checks cudaGetLastError
    (void)cudaGetLastError();
    return MSA_ERR_CUDA;
  }
  const cudaError_t e = msa::launch_block_lists(
      sel, d->batch * d->h_kv, d->n_q, d->q_pos0, msa_num_blocks(d), msa_query_window(d),
      blk_offsets, entries, entry_pos, total, ws, dev_err, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}
