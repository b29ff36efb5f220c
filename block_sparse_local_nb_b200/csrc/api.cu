// C ABI of the library (declared in include/nb.h): host-side argument
// validation, device check and dispatch to the kernel launchers.  Everything
// here runs on the host before any launch, so an invalid call launches nothing.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "../../include/nb.h"
#include "nb_internal.h"

namespace {

constexpr int kMaxDevices = 64;
// Per-device cache: 0 = unknown, 1 = sm_100 (supported), -1 = other.
int g_device_ok[kMaxDevices];

// Device word where kernels record the first wait-timeout code (0 = none),
// and its device address per device (looked up once).
__device__ int g_kernel_error;
std::mutex g_err_mutex;
int* g_err_addr[kMaxDevices];

int* error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_err_mutex);
  if (g_err_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_kernel_error) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_err_addr[dev] = static_cast<int*>(p);
  }
  return g_err_addr[dev];
}

nb_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return NB_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return NB_ERR_DEVICE;
  int state = __atomic_load_n(&g_device_ok[dev], __ATOMIC_RELAXED);
  if (state == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return NB_ERR_CUDA;
    state = (major == 10 && minor == 0) ? 1 : -1;
    __atomic_store_n(&g_device_ok[dev], state, __ATOMIC_RELAXED);
  }
  return state == 1 ? NB_OK : NB_ERR_DEVICE;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape checks shared by forward and backward.
nb_status check_shape(int batch, int heads, int n, int d, int R, int dtype) {
  if (batch < 0 || heads < 0 || n < 0 || R < 0) return NB_ERR_INVALID_ARG;
  if (n % nb::kBlock != 0) return NB_ERR_INVALID_ARG;
  if (dtype != NB_F32 && dtype != NB_BF16) return NB_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return NB_ERR_UNSUPPORTED;
  if (heads > 65535 || batch > 65535) return NB_ERR_UNSUPPORTED;  // grid y / z limits
  // element count must fit comfortably in int64 and rows*d*4 in size_t
  const double elems = static_cast<double>(batch) * heads * n * d;
  if (elems > 9.0e15) return NB_ERR_INVALID_ARG;
  return NB_OK;
}

nb::AttnArgs make_args(const void* q, const void* k, const void* v, const void* o,
                       const void* dout, const float* lse, const int32_t* lengths, void* dq,
                       void* dk, void* dv, void* ws, int batch, int heads, int n, int d, int R,
                       bool causal) {
  nb::AttnArgs a;
  a.q = q; a.k = k; a.v = v; a.o = o; a.dout = dout;
  a.lse = const_cast<float*>(lse);
  a.lengths = lengths;
  a.dq = dq; a.dk = dk; a.dv = dv; a.workspace = ws;
  a.batch = batch; a.heads = heads; a.n = n; a.d = d; a.R = R;
  a.scale = static_cast<float>(1.0 / sqrt(static_cast<double>(d)));
  a.causal = causal;
  a.err = error_word();
  return a;
}

nb_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                   const int32_t* lengths, int batch, int heads, int n, int d, int R, int dtype,
                   void* stream, bool causal) {
  nb_status st = check_shape(batch, heads, n, d, R, dtype);
  if (st != NB_OK) return st;
  if (static_cast<int64_t>(batch) * heads * n == 0) return NB_OK;
  if (!q || !k || !v || !o) return NB_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (lse && !aligned16(lse)) || (lengths && (reinterpret_cast<uintptr_t>(lengths) & 3u)))
    return NB_ERR_MISALIGNED;
  st = check_device();
  if (st != NB_OK) return st;
  nb::AttnArgs a = make_args(q, k, v, o, nullptr, lse, lengths, nullptr, nullptr, nullptr,
                             nullptr, batch, heads, n, d, R, causal);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e =
      dtype == NB_F32 ? nb::launch_attn_fwd_f32(a, s) : nb::launch_attn_fwd_bf16_tc(a, s);
  return e == cudaSuccess ? NB_OK : NB_ERR_CUDA;
}

// Pointer checks of the backward (null -> invalid, alignment).
nb_status bwd_pointers(const void* q, const void* k, const void* v, const void* o,
                       const void* dout, const float* lse, const int32_t* lengths, void* dq,
                       void* dk, void* dv) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return NB_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (lengths && (reinterpret_cast<uintptr_t>(lengths) & 3u)))
    return NB_ERR_MISALIGNED;
  return NB_OK;
}

nb_status attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                   const float* lse, const int32_t* lengths, void* dq, void* dk, void* dv,
                   void* workspace, size_t workspace_bytes, int batch, int heads, int n, int d,
                   int R, int dtype, void* stream, bool causal) {
  nb_status st = check_shape(batch, heads, n, d, R, dtype);
  if (st != NB_OK) return st;
  if (static_cast<int64_t>(batch) * heads * n == 0) return NB_OK;
  if (dtype != NB_BF16) return NB_ERR_UNSUPPORTED;
  st = bwd_pointers(q, k, v, o, dout, lse, lengths, dq, dk, dv);
  if (st != NB_OK) return st;
  const int64_t rows = static_cast<int64_t>(batch) * heads * n;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_bytes < nb::bwd_workspace_bytes(rows, d))
    return NB_ERR_WORKSPACE;
  st = check_device();
  if (st != NB_OK) return st;
  nb::AttnArgs a = make_args(q, k, v, o, dout, lse, lengths, dq, dk, dv, workspace, batch, heads,
                             n, d, R, causal);
  cudaError_t e = nb::launch_attn_bwd_bf16(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NB_OK : NB_ERR_CUDA;
}

}  // namespace

namespace nb {

nb_status bwd_host_checks(int batch, int heads, int n, int d, int R, int dtype) {
  const nb_status st = check_shape(batch, heads, n, d, R, dtype);
  if (st != NB_OK) return st;
  if (static_cast<int64_t>(batch) * heads * n == 0) return NB_OK;
  return dtype == NB_BF16 ? NB_OK : NB_ERR_UNSUPPORTED;
}

nb_status bwd_pointer_checks(const void* q, const void* k, const void* v, const void* o,
                             const void* dout, const float* lse, const int32_t* lengths,
                             void* dq, void* dk, void* dv) {
  return bwd_pointers(q, k, v, o, dout, lse, lengths, dq, dk, dv);
}

nb_status device_check() { return check_device(); }

}  // namespace nb

extern "C" {

const char* nb_status_string(int status) {
  switch (status) {
    case NB_OK: return "NB_OK";
    case NB_ERR_INVALID_ARG: return "NB_ERR_INVALID_ARG: invalid argument";
    case NB_ERR_UNSUPPORTED: return "NB_ERR_UNSUPPORTED: unsupported configuration";
    case NB_ERR_MISALIGNED: return "NB_ERR_MISALIGNED: pointer not 16-byte aligned";
    case NB_ERR_CUDA: return "NB_ERR_CUDA: CUDA runtime error";
    case NB_ERR_WORKSPACE: return "NB_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case NB_ERR_DEVICE: return "NB_ERR_DEVICE: current device is not sm_100";
    default: return "unknown nb_status";
  }
}

int nb_abi_version(void) { return 100; }

nb_status nb_kernel_error(int* code, int clear) {
  if (!code) return NB_ERR_INVALID_ARG;
  *code = 0;
  int* w = error_word();
  if (!w) return NB_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return NB_ERR_CUDA;
  if (cudaMemcpy(code, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return NB_ERR_CUDA;
  if (clear && *code != 0 && cudaMemset(w, 0, sizeof(int)) != cudaSuccess) return NB_ERR_CUDA;
  return NB_OK;
}

nb_status nb_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                      const int32_t* lengths, int batch, int heads, int n, int d, int R,
                      int dtype, void* stream) {
  return attn_fwd(q, k, v, o, lse, lengths, batch, heads, n, d, R, dtype, stream, false);
}

nb_status nb_attn_fwd_causal(const void* q, const void* k, const void* v, void* o, float* lse,
                             const int32_t* lengths, int batch, int heads, int n, int d, int R,
                             int dtype, void* stream) {
  return attn_fwd(q, k, v, o, lse, lengths, batch, heads, n, d, R, dtype, stream, true);
}

size_t nb_attn_bwd_workspace_size(int batch, int heads, int n, int d, int dtype) {
  if (check_shape(batch, heads, n, d, 0, dtype) != NB_OK) return 0;
  const int64_t rows = static_cast<int64_t>(batch) * heads * n;
  if (rows == 0) return 0;
  return nb::bwd_workspace_bytes(rows, d);
}

nb_status nb_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                      const void* dout, const float* lse, const int32_t* lengths, void* dq,
                      void* dk, void* dv, void* workspace, size_t workspace_bytes, int batch,
                      int heads, int n, int d, int R, int dtype, void* stream) {
  return attn_bwd(q, k, v, o, dout, lse, lengths, dq, dk, dv, workspace, workspace_bytes, batch,
                  heads, n, d, R, dtype, stream, false);
}

nb_status nb_attn_bwd_causal(const void* q, const void* k, const void* v, const void* o,
                             const void* dout, const float* lse, const int32_t* lengths, void* dq,
                             void* dk, void* dv, void* workspace, size_t workspace_bytes,
                             int batch, int heads, int n, int d, int R, int dtype, void* stream) {
  return attn_bwd(q, k, v, o, dout, lse, lengths, dq, dk, dv, workspace, workspace_bytes, batch,
                  heads, n, d, R, dtype, stream, true);
}

nb_status nb_tokenize_kmer(const uint8_t* seq, int64_t len, uint16_t* ids, uint8_t* packed,
                           int k, void* stream) {
  if (len < 0) return NB_ERR_INVALID_ARG;
  if (k < 1 || k > 7) return NB_ERR_UNSUPPORTED;
  if (ids && (reinterpret_cast<uintptr_t>(ids) & 1u)) return NB_ERR_MISALIGNED;
  if (len == 0 || (!ids && !packed)) return NB_OK;
  if (!seq) return NB_ERR_INVALID_ARG;
  if (len < k) ids = nullptr;  // no complete window: only the packed stream is written
  if (!ids && !packed) return NB_OK;
  nb_status st = check_device();
  if (st != NB_OK) return st;
  cudaError_t e =
      nb::launch_tokenize_kmer(seq, len, ids, packed, k, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NB_OK : NB_ERR_CUDA;
}

nb_status nb_tokenize_batch(const uint8_t* seqs, const int64_t* offsets, int batch, int k,
                            int64_t* input_ids, int32_t* lengths, int n_pad, void* stream) {
  if (batch < 0 || n_pad < 0 || n_pad % NB_BLOCK != 0) return NB_ERR_INVALID_ARG;
  if (k < 1 || k > 7 || batch > 65535) return NB_ERR_UNSUPPORTED;
  if (batch == 0) return NB_OK;
  if (!seqs || !offsets || (n_pad > 0 && !input_ids)) return NB_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(input_ids) & 15u) || (reinterpret_cast<uintptr_t>(offsets) & 7u) ||
      (reinterpret_cast<uintptr_t>(lengths) & 3u))
    return NB_ERR_MISALIGNED;
  if (n_pad == 0 && !lengths) return NB_OK;
  nb_status st = check_device();
  if (st != NB_OK) return st;
  cudaError_t e = nb::launch_tokenize_batch(seqs, offsets, batch, k, input_ids, lengths, n_pad,
                                            static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NB_OK : NB_ERR_CUDA;
}

nb_status nb_batch_ceiling(const int64_t* offsets, int batch, int k, int32_t* n_pad) {
  if (!n_pad || batch < 0 || (batch > 0 && !offsets)) return NB_ERR_INVALID_ARG;
  if (k < 1 || k > 7) return NB_ERR_UNSUPPORTED;
  int64_t windows = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t bases = offsets[b + 1] - offsets[b];
    const int64_t w = bases >= k ? bases - k + 1 : 0;
    if (w > windows) windows = w;
  }
  const int64_t ceil32 = (windows + NB_BLOCK - 1) / NB_BLOCK * NB_BLOCK;
  if (ceil32 > INT32_MAX) return NB_ERR_INVALID_ARG;
  *n_pad = static_cast<int32_t>(ceil32);
  return NB_OK;
}

}  // extern "C"
