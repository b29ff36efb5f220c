// Internal declarations shared by the C-ABI layer and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nb.h"

namespace nb {

constexpr int kBlock = 32;  // band block size B (NucleoByte page, section 3)

// Arguments of one attention call, already validated on the host.
struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* o;      // forward: output; backward: input
  const void* dout;   // backward only
  float* lse;         // forward: output (may be null); backward: input
  const int32_t* lengths;  // may be null = all full
  void* dq;
  void* dk;
  void* dv;
  void* workspace;
  int* err;           // device word receiving the first wait-timeout code (may be null)
  int batch, heads, n, d, R;
  float scale;        // 1/sqrt(d)
  bool causal;        // causal band: key blocks i - R..i of query block i, keys k <= q
};

size_t bwd_workspace_bytes(int64_t rows, int d);
__host__ __device__ inline int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

// TMA map over a [heads_total][n][d] bf16 tensor with 128-byte swizzle and a
// box of 64 columns x box_rows rows.
bool make_tmap_bf16_rows(CUtensorMap* m, const void* base, int d, int64_t n, int64_t heads_total,
                         int box_rows);
// Same for bf16 (box 64 columns) or fp32 tensors with a box of box_cols x box_rows
// (box_cols * element size must be 128 bytes for the swizzle).
bool make_tmap_rows(CUtensorMap* m, const void* base, bool f32, int d, int64_t n,
                    int64_t heads_total, int box_cols, int box_rows);
int num_sms();  // SM count of the current device (cached)

// Backward workspace: [-D: rows fp32][-lse*log2(e): rows fp32][dQ accumulator: rows*d fp32],
// each region 256-byte aligned.
struct BwdWorkspace {
  float* D;      // negated row term -D_i
  float* nlse2;
  float* dqacc;
};
__host__ __device__ inline BwdWorkspace bwd_workspace(void* ws, int64_t rows) {
  BwdWorkspace w;
  uint8_t* p = static_cast<uint8_t*>(ws);
  w.D = reinterpret_cast<float*>(p);
  w.nlse2 = reinterpret_cast<float*>(p + align_up(rows * 4, 256));
  w.dqacc = reinterpret_cast<float*>(p + 2 * align_up(rows * 4, 256));
  return w;
}
cudaError_t launch_bwd_main_tc(const AttnArgs& a, int64_t rows, cudaStream_t stream);
// d = 128 main kernel (64-query chunks; attn_bwd_tc_d128.cu)
cudaError_t launch_bwd_main_tc_d128(const AttnArgs& a, int64_t rows, cudaStream_t stream);

// Programmatic dependent launch.  Every kernel of this library is launched
// with it: a kernel may begin (set up barriers, tensor memory, descriptor
// prefetches) while the previous kernel on the stream is finishing, and
// executes pdl_wait() in every thread before its first access to global memory
// that earlier work on the stream may write or read.  pdl_trigger() lets the
// next kernel launch early; it never orders memory.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, const Args&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Host-side argument checks of the C ABI, shared by its entry points (api.cu).
nb_status bwd_host_checks(int batch, int heads, int n, int d, int R, int dtype);  // shape, dtype
nb_status bwd_pointer_checks(const void* q, const void* k, const void* v, const void* o,
                             const void* dout, const float* lse, const int32_t* lengths,
                             void* dq, void* dk, void* dv);  // null pointers, alignment
nb_status device_check();  // the current device is an sm_100 GPU

cudaError_t launch_tokenize_kmer(const uint8_t* seq, int64_t len, uint16_t* ids, uint8_t* packed,
                                 int k, cudaStream_t stream);
cudaError_t launch_tokenize_batch(const uint8_t* seqs, const int64_t* offsets, int batch, int k,
                                  int64_t* ids, int32_t* lengths, int n_pad, cudaStream_t stream);
cudaError_t launch_attn_fwd_f32(const AttnArgs& a, cudaStream_t stream);
cudaError_t launch_attn_fwd_bf16_tc(const AttnArgs& a, cudaStream_t stream);
cudaError_t launch_attn_bwd_bf16(const AttnArgs& a, cudaStream_t stream);

}  // namespace nb
