// Internal declarations shared by the C-ABI layer and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

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
  int batch, heads, n, d, R;
  float scale;        // 1/sqrt(d)
};

// Workspace layout of the backward: [row term D: rows fp32][dQ accumulator: rows*d fp32]
size_t bwd_workspace_bytes(int64_t rows, int d);
__host__ __device__ inline int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

cudaError_t launch_tokenize_kmer(const uint8_t* seq, int64_t len, uint16_t* ids, uint8_t* packed,
                                 int k, cudaStream_t stream);
cudaError_t launch_attn_fwd_f32(const AttnArgs& a, cudaStream_t stream);
cudaError_t launch_attn_fwd_bf16(const AttnArgs& a, cudaStream_t stream);
cudaError_t launch_attn_bwd_bf16(const AttnArgs& a, cudaStream_t stream);

}  // namespace nb
