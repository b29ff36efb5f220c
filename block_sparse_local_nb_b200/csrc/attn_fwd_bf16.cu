// Banded block-sparse local attention forward, bf16 in / fp32 accumulate
// (NucleoByte page, section 3 "Localized Block-Sparse Attention Matrix" and
// "Softmax Normalization & Online Numerical Stability").
//
// One CTA (8 warps) owns a query tile of four consecutive query blocks (128
// rows) of one (batch, head).  The union of their bands is the key-block
// window [4t - R, 4t + 3 + R]; its key and value blocks stream through a
// three-stage cp.async ring in shared memory, so each block is fetched once per
// tile and shared by every query block whose band contains it.  Warp w owns 16
// query rows of query block 4t + w/2 and skips key blocks outside that block's
// band.  Per 32-key block: S = Q K^T on tensor cores (m16n8k16), then the page's
// online update in base 2 (running max m, running sum l, O *= 2^(m_old -
// m_new)), then O += P V with P rounded to bf16.  Rows and keys at or past the
// sequence length are masked; padding rows get O = 0 and lse = -inf.
#include <math.h>

#include "nb_internal.h"
#include "warp_mma.cuh"

namespace nb {
namespace {

constexpr int kWarps = 8;
constexpr int kTileRows = 16 * kWarps;  // 128 query rows = 4 query blocks
constexpr int kStages = 3;

template <int D>
struct FwdSmem {
  static constexpr int kTileBytes = kBlock * D * 2;        // one 32-row block
  static constexpr int kQBytes = kTileRows * D * 2;
  static constexpr int kBytes = kQBytes + kStages * 2 * kTileBytes;
};

template <int D>
__device__ __forceinline__ void load_rows_async(uint32_t dst, const __nv_bfloat16* src,
                                                int rows, int valid_rows, int tid, int nthreads) {
  constexpr int CPR = D / 8;  // 16-byte chunks per row
  for (int idx = tid; idx < rows * CPR; idx += nthreads) {
    const int r = idx / CPR, c = idx % CPR;
    const bool ok = r < valid_rows;
    cp_async16(dst + tile_off<D>(r, c), ok ? src + (int64_t)r * D + c * 8 : src, ok);
  }
}

template <int D>
__global__ void __launch_bounds__(256) attn_fwd_bf16_kernel(AttnArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sKV = sQ + FwdSmem<D>::kQBytes;
  constexpr int TB = FwdSmem<D>::kTileBytes;

  const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int n = a.n, nb = n / kBlock;
  int L = a.lengths ? a.lengths[b] : n;
  L = min(max(L, 0), n);
  const int64_t head = ((int64_t)b * a.heads + h) * n;
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q) + head * D;
  const __nv_bfloat16* kp = static_cast<const __nv_bfloat16*>(a.k) + head * D;
  const __nv_bfloat16* vp = static_cast<const __nv_bfloat16*>(a.v) + head * D;
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(const_cast<void*>(a.o)) + head * D;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row0 = tile * kTileRows;
  const int rows_here = min(kTileRows, n - row0);

  if (row0 >= L) {  // every row of the tile is padding
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int idx = tid; idx < rows_here * (D / 8); idx += blockDim.x)
      reinterpret_cast<uint4*>(o + (int64_t)row0 * D)[idx] = z;
    if (a.lse)
      for (int r = tid; r < rows_here; r += blockDim.x) a.lse[head + row0 + r] = -INFINITY;
    return;
  }

  const int qb_first = tile * 4;
  const int qb_last = min(qb_first + 3, nb - 1);
  const int jlast = (L - 1) / kBlock;
  const int J0 = max(0, qb_first - a.R);
  const int J1 = min(min(qb_last + a.R, nb - 1), jlast);
  const int nj = J1 - J0 + 1;

  load_rows_async<D>(sQ, q + (int64_t)row0 * D, kTileRows, rows_here, tid, blockDim.x);
  cp_async_commit();
#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < nj) {
      const int j = J0 + s;
      const uint32_t dst = sKV + s * 2 * TB;
      load_rows_async<D>(dst, kp + (int64_t)j * kBlock * D, kBlock, kBlock, tid, blockDim.x);
      load_rows_async<D>(dst + TB, vp + (int64_t)j * kBlock * D, kBlock, kBlock, tid, blockDim.x);
    }
    cp_async_commit();
  }

  const int qb = qb_first + (warp >> 1);
  const bool active = qb <= qb_last && qb * kBlock < L;
  const int g = lane >> 2, tq = lane & 3;
  const int wrow = warp * 16;  // first tile row of this warp
  const float sl2 = a.scale * 1.4426950408889634f;  // scores in base-2 units

  uint32_t qf[D / 16][4];
  float acc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};

  cp_async_wait<kStages - 1>();  // Q tile landed
  __syncthreads();
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    ldsm_x4(qf[kk], sQ + tile_off<D>(wrow + (lane & 15), kk * 2 + (lane >> 4)));

  for (int it = 0; it < nj; ++it) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    {  // refill the stage freed by the previous iteration
      const int nxt = it + kStages - 1;
      if (nxt < nj) {
        const int j = J0 + nxt;
        const uint32_t dst = sKV + (nxt % kStages) * 2 * TB;
        load_rows_async<D>(dst, kp + (int64_t)j * kBlock * D, kBlock, kBlock, tid, blockDim.x);
        load_rows_async<D>(dst + TB, vp + (int64_t)j * kBlock * D, kBlock, kBlock, tid,
                           blockDim.x);
      }
      cp_async_commit();
    }
    const int j = J0 + it;
    if (!active || abs(qb - j) > a.R) continue;
    const uint32_t sK = sKV + (it % kStages) * 2 * TB;
    const uint32_t sV = sK + TB;

    float s[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        uint32_t r[4];
        ldsm_x4(r, sK + tile_off<D>(np * 16 + (lane & 7) + ((lane >> 4) << 3),
                                    kk * 2 + ((lane >> 3) & 1)));
        mma_16816(s[2 * np], qf[kk], r[0], r[1]);
        mma_16816(s[2 * np + 1], qf[kk], r[2], r[3]);
      }
    }
    // scale to base 2, mask keys at or past the length, running max per row
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = j * kBlock + nt * 8 + tq * 2 + (e & 1);
        float x = s[nt][e] * sl2;
        x = key < L ? x : -INFINITY;
        s[nt][e] = x;
        mx[e >> 1] = fmaxf(mx[e >> 1], x);
      }
    float alpha[2];
#pragma unroll
    for (int rh = 0; rh < 2; ++rh) {
      mx[rh] = fmaxf(mx[rh], __shfl_xor_sync(0xffffffffu, mx[rh], 1));
      mx[rh] = fmaxf(mx[rh], __shfl_xor_sync(0xffffffffu, mx[rh], 2));
      const float mnew = fmaxf(m[rh], mx[rh]);
      alpha[rh] = exp2f(m[rh] - mnew);
      m[rh] = mnew;
      l[rh] *= alpha[rh];
    }
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      acc[i][0] *= alpha[0]; acc[i][1] *= alpha[0];
      acc[i][2] *= alpha[1]; acc[i][3] *= alpha[1];
    }
    uint32_t pa[2][4];  // P as two m16n8k16 A fragments (keys 0-15, 16-31)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const float p0 = exp2f(s[nt][0] - m[0]), p1 = exp2f(s[nt][1] - m[0]);
      const float p2 = exp2f(s[nt][2] - m[1]), p3 = exp2f(s[nt][3] - m[1]);
      l[0] += p0 + p1;
      l[1] += p2 + p3;
      pa[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16(p0, p1);
      pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16(p2, p3);
    }
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        uint32_t r[4];
        ldsm_x4_t(r, sV + tile_off<D>(kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8,
                                      dp * 2 + (lane >> 4)));
        mma_16816(acc[2 * dp], pa[kk], r[0], r[1]);
        mma_16816(acc[2 * dp + 1], pa[kk], r[2], r[3]);
      }
    }
  }

  // epilogue: O = acc / l, staged through the (now free) Q tile for 16-byte stores
#pragma unroll
  for (int rh = 0; rh < 2; ++rh) {
    l[rh] += __shfl_xor_sync(0xffffffffu, l[rh], 1);
    l[rh] += __shfl_xor_sync(0xffffffffu, l[rh], 2);
  }
  float inv[2];
  bool rvalid[2];
#pragma unroll
  for (int rh = 0; rh < 2; ++rh) {
    const int r = row0 + wrow + g + rh * 8;
    rvalid[rh] = active && r < L;
    inv[rh] = rvalid[rh] ? 1.f / l[rh] : 0.f;
    if (a.lse && tq == 0 && wrow + g + rh * 8 < rows_here)
      a.lse[head + r] = rvalid[rh] ? (m[rh] + log2f(l[rh])) * 0.6931471805599453f : -INFINITY;
  }
  uint8_t* sOut = smem;  // reuse the Q tile (each warp touches only its own 16 rows)
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
#pragma unroll
    for (int rh = 0; rh < 2; ++rh) {
      const int r = wrow + g + rh * 8;
      *reinterpret_cast<uint32_t*>(sOut + tile_off<D>(r, i) + tq * 4) =
          pack_bf16(acc[i][2 * rh] * inv[rh], acc[i][2 * rh + 1] * inv[rh]);
    }
  }
  __syncwarp();
  constexpr int CPR = D / 8;
  for (int idx = lane; idx < 16 * CPR; idx += 32) {
    const int r = wrow + idx / CPR, c = idx % CPR;
    if (r < rows_here)
      *reinterpret_cast<uint4*>(o + (int64_t)(row0 + r) * D + c * 8) =
          *reinterpret_cast<const uint4*>(sOut + tile_off<D>(r, c));
  }
}

template <int D>
cudaError_t launch(const AttnArgs& a, cudaStream_t stream) {
  const int bytes = FwdSmem<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_bf16_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  dim3 grid((a.n + kTileRows - 1) / kTileRows, a.heads, a.batch);
  attn_fwd_bf16_kernel<D><<<grid, kWarps * 32, bytes, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_bf16(const AttnArgs& a, cudaStream_t stream) {
  return a.d == 64 ? launch<64>(a, stream) : launch<128>(a, stream);
}

}  // namespace nb
