// nb_attn_bwd_noalloc: the attention backward for callers that cannot
// allocate device memory themselves.
//
// nb_attn_bwd needs a caller-provided workspace (the per-row term D and the
// fp32 dQ accumulator).  Some callers have no way to provide one: a host
// program whose device memory is entirely owned by another allocator (a
// framework's caching allocator that has reserved the GPU), an embedding
// through a foreign-function interface that exposes no allocator, or a
// latency-critical loop in which cudaMalloc / cudaFree, which may synchronise
// the device, are not acceptable.  This entry point serves them from a fixed
// scratch array compiled into the library instead.
//
// The scratch is a file-scope __device__ array of NB_NOALLOC_SCRATCH_BYTES
// (64 MiB).  It occupies that much memory on every GPU where this library's
// code is loaded, until the process exits.  In host code its name is only a
// host-side stand-in, so its device address is looked up with
// cudaGetSymbolAddress once per device, on the first call made with that
// device current, and then passed to the kernels.  All calls share the one
// array: calls whose work overlaps on the GPU (other streams, other host
// threads) race on it and must be serialised by the caller.  The kernels
// rewrite every byte they read from it on each call (the row term and the
// zeroed dQ accumulator), so contents left by an earlier call do not matter.
//
// The checks run in this order, all on the host before the symbol lookup, so
// a rejected call neither launches nor loads the array: shape and dtype (as
// nb_attn_bwd), the scratch limit (NB_ERR_WORKSPACE), pointers (as
// nb_attn_bwd), the device (NB_ERR_DEVICE).
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/nb.h"
#include "nb_internal.h"

namespace {

constexpr size_t kScratchBytes = NB_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_bwd_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices];  // device address of g_bwd_scratch, per device

// Device address of the scratch array on the current device (set up once).
nb_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return NB_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return NB_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();  // the failed lookup's error, so an unrelated later call does not report it
      return NB_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return NB_OK;
}

}  // namespace

extern "C" NB_API nb_status nb_attn_bwd_noalloc(const void* q, const void* k, const void* v,
                                                const void* o, const void* dout, const float* lse,
                                                const int32_t* lengths, void* dq, void* dk,
                                                void* dv, int batch, int heads, int n, int d,
                                                int R, int dtype, void* stream) {
  nb_status st = nb::bwd_host_checks(batch, heads, n, d, R, dtype);
  if (st != NB_OK) return st;
  const size_t need = nb_attn_bwd_workspace_size(batch, heads, n, d, dtype);
  if (need == 0) return NB_OK;                      // empty problem: nothing to do
  if (need > kScratchBytes) return NB_ERR_WORKSPACE;  // beyond the built-in scratch
  st = nb::bwd_pointer_checks(q, k, v, o, dout, lse, lengths, dq, dk, dv);
  if (st != NB_OK) return st;
  st = nb::device_check();
  if (st != NB_OK) return st;
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != NB_OK) return st;
  return nb_attn_bwd(q, k, v, o, dout, lse, lengths, dq, dk, dv, scratch, kScratchBytes, batch,
                     heads, n, d, R, dtype, stream);
}
