// Banded block-sparse local attention backward, bf16 in / fp32 accumulate:
// the memory-bound row-term kernel before the tensor-core main kernel
// (attn_bwd_tc.cu), both on the caller's stream.  (NucleoByte page, section 3
// "Custom Backpropagation": the row term D_i = sum_k dO_ik O_ik.)
//
//  1. rowterm: per row, D = rowsum(dO * O) and -lse * log2(e) (both 0 / -inf on
//     padding rows, so padding queries get P = 0 in the main kernel); dQ = 0 on
//     the rows of query blocks that hold no valid query (no key tile adds to
//     them); the per-block arrival and completion counters of the dQ
//     accumulation set to 0.
//  2. main (attn_bwd_tc.cu): dK, dV, and dQ accumulated per query block in the
//     fp32 workspace, the last key tile of a block writing its bf16 dQ.
#include <math.h>

#include "nb_internal.h"
#include "sm100.cuh"

namespace nb {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

template <int D>
__global__ void __launch_bounds__(256) bwd_rowterm_kernel(AttnArgs a, int64_t rows) {
  constexpr int TPR = D / 8;  // threads per row, 8 elements (16 bytes) each
  pdl_trigger();
  pdl_wait();
  const BwdWorkspace w = bwd_workspace(a.workspace, rows, D);
  const int64_t gt = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t row = gt / TPR;
  const int part = static_cast<int>(gt % TPR);
  const bool in = row < rows;
  bool valid = false;
  float acc = 0.f;
  if (in) {
    const int64_t bh = row / a.n;
    const int qi = static_cast<int>(row % a.n);
    int L = a.lengths ? a.lengths[bh / a.heads] : a.n;
    L = min(max(L, 0), a.n);
    valid = qi < L;
    if (valid) {
      const uint4 ov = *reinterpret_cast<const uint4*>(
          static_cast<const __nv_bfloat16*>(a.o) + row * D + part * 8);
      const uint4 dv = *reinterpret_cast<const uint4*>(
          static_cast<const __nv_bfloat16*>(a.dout) + row * D + part * 8);
      const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
      const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 of = __bfloat1622float2(o2[i]);
        const float2 df = __bfloat1622float2(d2[i]);
        acc = fmaf(of.x, df.x, acc);
        acc = fmaf(of.y, df.y, acc);
      }
    } else if ((qi & ~(kBlock - 1)) >= L) {  // a block with no valid query: dQ = 0 here
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.dq) + row * D + part * 8) =
          make_uint4(0, 0, 0, 0);
    }
  }
#pragma unroll
  for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (in && part == 0) {
    w.D[row] = -acc;  // stored negated: the main kernel forms dP + (-D)
    w.nlse2[row] = valid ? -a.lse[row] * kLog2e : -INFINITY;
    if ((row & (kBlock - 1)) == 0) {  // one thread per query block clears its counters
      w.arrive[row / kBlock] = 0;
      w.done[row / kBlock] = 0;
    }
  }
}

template <int D>
cudaError_t run(const AttnArgs& a, cudaStream_t stream) {
  const int64_t rows = (int64_t)a.batch * a.heads * a.n;
  const int64_t threads = rows * (D / 8);
  const int64_t blocks = (threads + 255) / 256;
  cudaError_t e =
      launch_pdl(bwd_rowterm_kernel<D>, dim3((unsigned)blocks), dim3(256), 0, stream, a, rows);
  if (e != cudaSuccess) return e;
  return launch_bwd_main_tc(a, rows, stream);
}

}  // namespace

size_t bwd_workspace_bytes(int64_t rows, int d) {
  return static_cast<size_t>(2 * align_up(rows * 4, 256) + align_up(rows * d * 4, 256) +
                             2 * align_up(rows / kBlock * 4, 256));
}

cudaError_t launch_attn_bwd_bf16(const AttnArgs& a, cudaStream_t stream) {
  return a.d == 64 ? run<64>(a, stream) : run<128>(a, stream);
}

}  // namespace nb
