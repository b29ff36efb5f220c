// Banded block-sparse local attention backward, bf16 in / fp32 accumulate:
// the two memory-bound kernels around the tensor-core main kernel
// (attn_bwd_tc.cu), all on the caller's stream.  (NucleoByte page, section 3
// "Custom Backpropagation": the row term D_i = sum_k dO_ik O_ik.)
//
//  1. rowterm: per row, D = rowsum(dO * O) and -lse * log2(e) (both 0 / -inf on
//     padding rows, so padding queries get P = 0 in the main kernel), and zero
//     the fp32 dQ accumulator.
//  2. main (attn_bwd_tc.cu): dK, dV and the dQ accumulation.
//  3. dq_out: dQ = bf16(accumulator / sqrt(d)) on valid rows, 0 on padding rows.
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
  const BwdWorkspace w = bwd_workspace(a.workspace, rows);
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
    }
    if (valid) {  // padding rows of the accumulator are never read
      float4* z = reinterpret_cast<float4*>(w.dqacc + row * D + part * 8);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
#pragma unroll
  for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (in && part == 0) {
    w.D[row] = -acc;  // stored negated: the main kernel forms dP + (-D)
    w.nlse2[row] = valid ? -a.lse[row] * kLog2e : -INFINITY;
  }
}

template <int D>
__global__ void __launch_bounds__(256) bwd_dq_out_kernel(AttnArgs a, int64_t rows) {
  pdl_trigger();
  pdl_wait();
  const float* dqacc = bwd_workspace(a.workspace, rows).dqacc;
  const int64_t nvec = rows * D / 8;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < nvec;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = idx / (D / 8);
    const int64_t bh = row / a.n;
    int L = a.lengths ? a.lengths[bh / a.heads] : a.n;
    L = min(max(L, 0), a.n);
    if (row - bh * a.n >= L) {  // padding row: dQ = 0, accumulator not read
      reinterpret_cast<uint4*>(a.dq)[idx] = make_uint4(0, 0, 0, 0);
      continue;
    }
    const float4 x = reinterpret_cast<const float4*>(dqacc)[2 * idx];
    const float4 y = reinterpret_cast<const float4*>(dqacc)[2 * idx + 1];
    uint4 out;
    out.x = pack_bf16(x.x * a.scale, x.y * a.scale);
    out.y = pack_bf16(x.z * a.scale, x.w * a.scale);
    out.z = pack_bf16(y.x * a.scale, y.y * a.scale);
    out.w = pack_bf16(y.z * a.scale, y.w * a.scale);
    reinterpret_cast<uint4*>(a.dq)[idx] = out;
  }
}

template <int D>
cudaError_t run(const AttnArgs& a, cudaStream_t stream) {
  const int64_t rows = (int64_t)a.batch * a.heads * a.n;
  {
    const int64_t threads = rows * (D / 8);
    const int64_t blocks = (threads + 255) / 256;
    cudaError_t e = launch_pdl(bwd_rowterm_kernel<D>, dim3((unsigned)blocks), dim3(256), 0, stream, a, rows);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = launch_bwd_main_tc(a, rows, stream);
  if (e != cudaSuccess) return e;
  {
    const int64_t nvec = rows * D / 8;
    int64_t blocks = (nvec + 255) / 256;
    if (blocks > 148 * 64) blocks = 148 * 64;
    e = launch_pdl(bwd_dq_out_kernel<D>, dim3((unsigned)blocks), dim3(256), 0, stream, a, rows);
  }
  return e;
}

}  // namespace

size_t bwd_workspace_bytes(int64_t rows, int d) {
  return static_cast<size_t>(2 * align_up(rows * 4, 256) + align_up(rows * d * 4, 256));
}

cudaError_t launch_attn_bwd_bf16(const AttnArgs& a, cudaStream_t stream) {
  return a.d == 64 ? run<64>(a, stream) : run<128>(a, stream);
}

}  // namespace nb
