// Banded block-sparse local attention forward in fp32 on the CUDA cores
// (NucleoByte page, section 3: band |i - j| <= R over blocks of 32, scores
// Q K^T / sqrt(d), online softmax with running max m, running sum l and
// running output, rescaled by exp(m_old - m_new) at each active key block).
//
// fp32 inputs need ~1e-6 relative accuracy, which TF32 tensor cores do not
// give, so this path uses FFMA.  One CTA of 128 threads owns one query block
// (32 rows): four threads per row, each holding d/4 interleaved dimensions of
// the query and of the output accumulator.  The key and value blocks of the
// band are staged through shared memory one block at a time.  With the causal
// band (a.causal) the window is blocks qb - R .. qb and keys after the query
// are masked.
#include <math.h>

#include "nb_internal.h"

namespace nb {
namespace {

template <int D>
__global__ void __launch_bounds__(128) attn_fwd_f32_kernel(AttnArgs a) {
  constexpr int DPT = D / 4;  // dimensions per thread
  __shared__ __align__(16) float Ks[kBlock][D];
  __shared__ __align__(16) float Vs[kBlock][D];

  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int n = a.n, nb = n / kBlock;
  int L = a.lengths ? a.lengths[b] : n;
  L = min(max(L, 0), n);
  const int64_t head = ((int64_t)b * a.heads + h) * n;  // first row of this (b, h)
  const float* q = static_cast<const float*>(a.q) + head * D;
  const float* kp = static_cast<const float*>(a.k) + head * D;
  const float* vp = static_cast<const float*>(a.v) + head * D;
  float* o = static_cast<float*>(const_cast<void*>(a.o)) + head * D;

  const int row = threadIdx.x >> 2, sub = threadIdx.x & 3;
  const int qrow = qb * kBlock + row;

  if (qb * kBlock >= L) {  // the whole query block is padding
#pragma unroll
    for (int i = 0; i < DPT; ++i) o[(int64_t)qrow * D + sub + 4 * i] = 0.f;
    if (a.lse && sub == 0) a.lse[head + qrow] = -INFINITY;
    return;
  }

  float qv[DPT], acc[DPT];
#pragma unroll
  for (int i = 0; i < DPT; ++i) {
    qv[i] = q[(int64_t)qrow * D + sub + 4 * i] * a.scale;
    acc[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;

  const int jlast = (L - 1) / kBlock;  // last key block holding a valid key
  const int j0 = max(0, qb - a.R), j1 = min(min(nb - 1, qb + (a.causal ? 0 : a.R)), jlast);
  for (int j = j0; j <= j1; ++j) {
    const float4* ksrc = reinterpret_cast<const float4*>(kp + (int64_t)j * kBlock * D);
    const float4* vsrc = reinterpret_cast<const float4*>(vp + (int64_t)j * kBlock * D);
    for (int idx = threadIdx.x; idx < kBlock * D / 4; idx += 128) {
      reinterpret_cast<float4*>(&Ks[0][0])[idx] = ksrc[idx];
      reinterpret_cast<float4*>(&Vs[0][0])[idx] = vsrc[idx];
    }
    __syncthreads();
    float s[kBlock];
    float mblk = -INFINITY;
#pragma unroll
    for (int kk = 0; kk < kBlock; ++kk) {
      float part = 0.f;
#pragma unroll
      for (int i = 0; i < DPT; ++i) part = fmaf(qv[i], Ks[kk][sub + 4 * i], part);
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      part += __shfl_xor_sync(0xffffffffu, part, 2);
      const int key = j * kBlock + kk;  // keys past the length (or, causal, after the query) masked
      s[kk] = (key < L && (!a.causal || key <= qrow)) ? part : -INFINITY;
      mblk = fmaxf(mblk, s[kk]);
    }
    const float mnew = fmaxf(m, mblk);
    const float alpha = expf(m - mnew);
    l *= alpha;
#pragma unroll
    for (int i = 0; i < DPT; ++i) acc[i] *= alpha;
#pragma unroll
    for (int kk = 0; kk < kBlock; ++kk) {
      const float p = expf(s[kk] - mnew);
      l += p;
#pragma unroll
      for (int i = 0; i < DPT; ++i) acc[i] = fmaf(p, Vs[kk][sub + 4 * i], acc[i]);
    }
    m = mnew;
    __syncthreads();
  }

  const bool valid = qrow < L;
  const float inv = valid ? 1.f / l : 0.f;
#pragma unroll
  for (int i = 0; i < DPT; ++i) o[(int64_t)qrow * D + sub + 4 * i] = acc[i] * inv;
  if (a.lse && sub == 0) a.lse[head + qrow] = valid ? m + logf(l) : -INFINITY;
}

}  // namespace

cudaError_t launch_attn_fwd_f32(const AttnArgs& a, cudaStream_t stream) {
  dim3 grid(a.n / kBlock, a.heads, a.batch);
  if (a.d == 64)
    attn_fwd_f32_kernel<64><<<grid, 128, 0, stream>>>(a);
  else
    attn_fwd_f32_kernel<128><<<grid, 128, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace nb
