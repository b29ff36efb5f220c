// Banded block-sparse local attention backward, bf16 in / fp32 accumulate
// (NucleoByte page, section 3 "Custom Backpropagation": row term
// D_i = sum_k dO_ik O_ik, softmax gradient dS_ij = P_ij (dO_i V_j^T - D_i), and
// accumulation of gradients of shared key/value blocks with atomic adds).
//
// Three launches on the caller's stream:
//  1. rowterm:  D = rowsum(dO * O) (fp32, 0 on padding rows) and zero the fp32
//               dQ accumulator; both live in the caller's workspace.
//  2. main:     one CTA (4 warps) per key tile of two key blocks (64 keys).  The
//               band is symmetric, so the tile's dK and dV need only query blocks
//               [2t - R, 2t + 1 + R]; they stream through a two-stage cp.async
//               ring (Q, dO, lse, D) and dK, dV accumulate in registers with no
//               atomics (deterministic).  P is recomputed from the stored
//               log-sum-exp: P = 2^(S log2e - lse log2e).  Per query block the CTA
//               forms dS^T in shared memory and adds dQ_i += dS K into the fp32
//               accumulator with vector reductions (the page's atomicAdd).
//  3. dq_out:   dQ = bf16(accumulator / sqrt(d)).
#include <math.h>

#include "nb_internal.h"
#include "warp_mma.cuh"

namespace nb {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------- 1. rowterm
template <int D>
__global__ void __launch_bounds__(256) bwd_rowterm_kernel(AttnArgs a, int64_t rows) {
  constexpr int TPR = D / 8;  // threads per row, 8 elements (16 bytes) each
  float* Dvec = static_cast<float*>(a.workspace);
  float* dqacc = reinterpret_cast<float*>(static_cast<uint8_t*>(a.workspace) +
                                          align_up(rows * 4, 256));
  const int64_t gt = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t row = gt / TPR;
  const int part = static_cast<int>(gt % TPR);
  const bool in = row < rows;
  float acc = 0.f;
  if (in) {
    const int64_t bh = row / a.n;
    const int qi = static_cast<int>(row % a.n);
    int L = a.lengths ? a.lengths[bh / a.heads] : a.n;
    L = min(max(L, 0), a.n);
    if (qi < L) {
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
    float4* z = reinterpret_cast<float4*>(dqacc + row * D + part * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (in && part == 0) Dvec[row] = acc;
}

// ------------------------------------------------------------------ 2. main
constexpr int kKeyRows = 64;  // keys per CTA (two key blocks)
constexpr int kBwdStages = 2;

template <int D>
struct BwdSmem {
  static constexpr int kKV = kKeyRows * D * 2;       // one of K, V
  static constexpr int kQ = kBlock * D * 2;          // one of Q_i, dO_i
  static constexpr int kStage = 2 * kQ + 2 * kBlock * 4;  // Q, dO, lse, D
  static constexpr int kDS = kKeyRows * kBlock * 2;  // dS^T tile, bf16
  static constexpr int kBytes = 2 * kKV + kBwdStages * kStage + kDS;
};

// dS^T tile: 64 key rows x 32 query columns (4 chunks of 16 bytes per row),
// chunk swizzled by (row >> 1) & 3 so transposed ldmatrix reads are conflict-free.
__device__ __forceinline__ uint32_t ds_off(int key, int chunk) {
  return static_cast<uint32_t>(key * 64 + ((chunk ^ ((key >> 1) & 3)) << 4));
}

template <int D>
__device__ __forceinline__ void load_rows(uint32_t dst, const __nv_bfloat16* src, int rows,
                                          int valid_rows, int tid) {
  constexpr int CPR = D / 8;
  for (int idx = tid; idx < rows * CPR; idx += 128) {
    const int r = idx / CPR, c = idx % CPR;
    const bool ok = r < valid_rows;
    cp_async16(dst + tile_off<D>(r, c), ok ? src + (int64_t)r * D + c * 8 : src, ok);
  }
}

template <int D>
__global__ void __launch_bounds__(128) bwd_main_kernel(AttnArgs a, int64_t rows) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sK = smem_u32(smem);
  const uint32_t sV = sK + BwdSmem<D>::kKV;
  const uint32_t sStage0 = sV + BwdSmem<D>::kKV;
  const uint32_t sDS = sStage0 + kBwdStages * BwdSmem<D>::kStage;
  uint8_t* stage_ptr0 = smem + 2 * BwdSmem<D>::kKV;

  const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int n = a.n, nb = n / kBlock;
  int L = a.lengths ? a.lengths[b] : n;
  L = min(max(L, 0), n);
  const int64_t head = ((int64_t)b * a.heads + h) * n;
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q) + head * D;
  const __nv_bfloat16* kp = static_cast<const __nv_bfloat16*>(a.k) + head * D;
  const __nv_bfloat16* vp = static_cast<const __nv_bfloat16*>(a.v) + head * D;
  const __nv_bfloat16* dop = static_cast<const __nv_bfloat16*>(a.dout) + head * D;
  const float* lse = a.lse + head;
  const float* Dvec = static_cast<const float*>(a.workspace) + head;
  float* dqacc = reinterpret_cast<float*>(static_cast<uint8_t*>(a.workspace) +
                                          align_up(rows * 4, 256)) + head * D;
  __nv_bfloat16* dkp = static_cast<__nv_bfloat16*>(a.dk) + head * D;
  __nv_bfloat16* dvp = static_cast<__nv_bfloat16*>(a.dv) + head * D;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int key0 = tile * kKeyRows;
  const int keys_here = min(kKeyRows, n - key0);

  if (key0 >= L) {  // every key of the tile is padding: zero dK, dV
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int idx = tid; idx < keys_here * (D / 8); idx += 128) {
      reinterpret_cast<uint4*>(dkp + (int64_t)key0 * D)[idx] = z;
      reinterpret_cast<uint4*>(dvp + (int64_t)key0 * D)[idx] = z;
    }
    return;
  }

  const int kb_first = tile * 2;
  const int kb_last = min(kb_first + 1, nb - 1);
  const int ilast = (L - 1) / kBlock;
  const int I0 = max(0, kb_first - a.R);
  const int I1 = min(min(kb_last + a.R, nb - 1), ilast);
  const int ni = I1 - I0 + 1;

  load_rows<D>(sK, kp + (int64_t)key0 * D, kKeyRows, keys_here, tid);
  load_rows<D>(sV, vp + (int64_t)key0 * D, kKeyRows, keys_here, tid);
  auto load_stage = [&](int s, int i) {
    const uint32_t base = sStage0 + s * BwdSmem<D>::kStage;
    load_rows<D>(base, q + (int64_t)i * kBlock * D, kBlock, kBlock, tid);
    load_rows<D>(base + BwdSmem<D>::kQ, dop + (int64_t)i * kBlock * D, kBlock, kBlock, tid);
    if (tid < 8) {
      cp_async16(base + 2 * BwdSmem<D>::kQ + tid * 16, lse + (int64_t)i * kBlock + tid * 4, true);
    } else if (tid < 16) {
      cp_async16(base + 2 * BwdSmem<D>::kQ + kBlock * 4 + (tid - 8) * 16,
                 Dvec + (int64_t)i * kBlock + (tid - 8) * 4, true);
    }
  };
  load_stage(0, I0);
  cp_async_commit();

  const int kb = kb_first + (warp >> 1);  // this warp's key block
  const bool kactive = kb <= kb_last && kb * kBlock < L;
  const int g = lane >> 2, tq = lane & 3;
  const int wkey = warp * 16;  // first tile key row of this warp
  const float sl2 = a.scale * kLog2e;

  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[i][e] = dv[i][e] = 0.f;

  // dQ split: warp -> query rows 16*(warp & 1).., dims (warp >> 1) * D/2 ..
  const int mt = warp & 1, dh = warp >> 1;

  for (int it = 0; it < ni; ++it) {
    const int i = I0 + it;
    if (it + 1 < ni) load_stage((it + 1) % kBwdStages, i + 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t sQ = sStage0 + (it % kBwdStages) * BwdSmem<D>::kStage;
    const uint32_t sdO = sQ + BwdSmem<D>::kQ;
    const float* lse_s = reinterpret_cast<const float*>(stage_ptr0 + (it % kBwdStages) * BwdSmem<D>::kStage +
                                                        2 * BwdSmem<D>::kQ);
    const float* D_s = lse_s + kBlock;

    const bool live = kactive && abs(kb - i) <= a.R;
    if (live) {
      // S^T = K_w Q_i^T and dP^T = V_w dO_i^T: 16 keys x 32 queries each
      float st[4][4], dpt[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) st[nt][e] = dpt[nt][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t ka[4], va[4];
        ldsm_x4(ka, sK + tile_off<D>(wkey + (lane & 15), kk * 2 + (lane >> 4)));
        ldsm_x4(va, sV + tile_off<D>(wkey + (lane & 15), kk * 2 + (lane >> 4)));
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          uint32_t r[4];
          const int qrow = np * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int qch = kk * 2 + ((lane >> 3) & 1);
          ldsm_x4(r, sQ + tile_off<D>(qrow, qch));
          mma_16816(st[2 * np], ka, r[0], r[1]);
          mma_16816(st[2 * np + 1], ka, r[2], r[3]);
          ldsm_x4(r, sdO + tile_off<D>(qrow, qch));
          mma_16816(dpt[2 * np], va, r[0], r[1]);
          mma_16816(dpt[2 * np + 1], va, r[2], r[3]);
        }
      }
      // P^T and dS^T (rows = keys, columns = queries)
      uint32_t pa[2][4], sa[2][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        float p[4], ds[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = nt * 8 + tq * 2 + (e & 1);
          const int key = key0 + wkey + g + (e >> 1) * 8;
          const int qi = i * kBlock + col;
          const bool vis = key < L && qi < L;
          const float pe = vis ? exp2f(st[nt][e] * sl2 - lse_s[col] * kLog2e) : 0.f;
          p[e] = pe;
          ds[e] = pe * (dpt[nt][e] - D_s[col]);
        }
        pa[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16(p[0], p[1]);
        pa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16(p[2], p[3]);
        sa[nt >> 1][(nt & 1) * 2 + 0] = pack_bf16(ds[0], ds[1]);
        sa[nt >> 1][(nt & 1) * 2 + 1] = pack_bf16(ds[2], ds[3]);
        // dS^T to shared memory for the dQ product
        uint8_t* dsb = smem + (sDS - sK);
        *reinterpret_cast<uint32_t*>(dsb + ds_off(wkey + g, nt) + tq * 4) =
            sa[nt >> 1][(nt & 1) * 2 + 0];
        *reinterpret_cast<uint32_t*>(dsb + ds_off(wkey + g + 8, nt) + tq * 4) =
            sa[nt >> 1][(nt & 1) * 2 + 1];
      }
      // dV += P^T dO_i ; dK += dS^T Q_i   (k dimension = 32 queries)
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
        for (int dp = 0; dp < D / 16; ++dp) {
          uint32_t r[4];
          const int qrow = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int dch = dp * 2 + (lane >> 4);
          ldsm_x4_t(r, sdO + tile_off<D>(qrow, dch));
          mma_16816(dv[2 * dp], pa[kk], r[0], r[1]);
          mma_16816(dv[2 * dp + 1], pa[kk], r[2], r[3]);
          ldsm_x4_t(r, sQ + tile_off<D>(qrow, dch));
          mma_16816(dk[2 * dp], sa[kk], r[0], r[1]);
          mma_16816(dk[2 * dp + 1], sa[kk], r[2], r[3]);
        }
      }
    } else {
      // keys outside query block i's band contribute nothing to dQ_i
      uint8_t* dsb = smem + (sDS - sK);
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        *reinterpret_cast<uint32_t*>(dsb + ds_off(wkey + g, nt) + tq * 4) = 0u;
        *reinterpret_cast<uint32_t*>(dsb + ds_off(wkey + g + 8, nt) + tq * 4) = 0u;
      }
    }
    __syncthreads();

    // dQ_i (32 x D) += dS (32 x 64) K_tile (64 x D), this warp's 16 rows x D/2 dims
    {
      float dq[D / 16][4];
#pragma unroll
      for (int nt = 0; nt < D / 16; ++nt) dq[nt][0] = dq[nt][1] = dq[nt][2] = dq[nt][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < kKeyRows / 16; ++kk) {
        uint32_t af[4];
        ldsm_x4_t(af, sDS + ds_off(kk * 16 + (lane & 7) + ((lane >> 4) << 3),
                                   mt * 2 + ((lane >> 3) & 1)));
#pragma unroll
        for (int dp = 0; dp < D / 32; ++dp) {
          uint32_t r[4];
          ldsm_x4_t(r, sK + tile_off<D>(kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8,
                                        dh * (D / 16) + dp * 2 + (lane >> 4)));
          mma_16816(dq[2 * dp], af, r[0], r[1]);
          mma_16816(dq[2 * dp + 1], af, r[2], r[3]);
        }
      }
#pragma unroll
      for (int rh = 0; rh < 2; ++rh) {
        const int qi = i * kBlock + mt * 16 + g + rh * 8;
        if (qi < L) {
          float* dst = dqacc + (int64_t)qi * D + dh * (D / 2) + tq * 2;
#pragma unroll
          for (int nt = 0; nt < D / 16; ++nt)
            red_add_v2(dst + nt * 8, dq[nt][2 * rh], dq[nt][2 * rh + 1]);
        }
      }
    }
  }

  // epilogue: dK *= 1/sqrt(d); zero rows past the length; stage through K/V tiles
  __syncthreads();  // all warps are done reading sK / sV
  uint8_t* oK = smem;
  uint8_t* oV = smem + BwdSmem<D>::kKV;
#pragma unroll
  for (int rh = 0; rh < 2; ++rh) {
    const int r = wkey + g + rh * 8;
    const bool ok = kactive && key0 + r < L;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      *reinterpret_cast<uint32_t*>(oK + tile_off<D>(r, nt) + tq * 4) =
          ok ? pack_bf16(dk[nt][2 * rh] * a.scale, dk[nt][2 * rh + 1] * a.scale) : 0u;
      *reinterpret_cast<uint32_t*>(oV + tile_off<D>(r, nt) + tq * 4) =
          ok ? pack_bf16(dv[nt][2 * rh], dv[nt][2 * rh + 1]) : 0u;
    }
  }
  __syncthreads();
  constexpr int CPR = D / 8;
  for (int idx = tid; idx < keys_here * CPR; idx += 128) {
    const int r = idx / CPR, c = idx % CPR;
    *reinterpret_cast<uint4*>(dkp + (int64_t)(key0 + r) * D + c * 8) =
        *reinterpret_cast<const uint4*>(oK + tile_off<D>(r, c));
    *reinterpret_cast<uint4*>(dvp + (int64_t)(key0 + r) * D + c * 8) =
        *reinterpret_cast<const uint4*>(oV + tile_off<D>(r, c));
  }
}

// ---------------------------------------------------------------- 3. dq_out
template <int D>
__global__ void __launch_bounds__(256) bwd_dq_out_kernel(AttnArgs a, int64_t rows) {
  const float* dqacc = reinterpret_cast<const float*>(static_cast<const uint8_t*>(a.workspace) +
                                                      align_up(rows * 4, 256));
  const int64_t nvec = rows * D / 8;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < nvec;
       idx += (int64_t)gridDim.x * blockDim.x) {
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
    bwd_rowterm_kernel<D><<<(unsigned)blocks, 256, 0, stream>>>(a, rows);
  }
  {
    const int bytes = BwdSmem<D>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(bwd_main_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    dim3 grid((a.n + kKeyRows - 1) / kKeyRows, a.heads, a.batch);
    bwd_main_kernel<D><<<grid, 128, bytes, stream>>>(a, rows);
  }
  {
    const int64_t nvec = rows * D / 8;
    int64_t blocks = (nvec + 255) / 256;
    if (blocks > 148 * 64) blocks = 148 * 64;
    bwd_dq_out_kernel<D><<<(unsigned)blocks, 256, 0, stream>>>(a, rows);
  }
  return cudaGetLastError();
}

}  // namespace

size_t bwd_workspace_bytes(int64_t rows, int d) {
  return static_cast<size_t>(align_up(rows * 4, 256) + align_up(rows * d * 4, 256));
}

cudaError_t launch_attn_bwd_bf16(const AttnArgs& a, cudaStream_t stream) {
  return a.d == 64 ? run<64>(a, stream) : run<128>(a, stream);
}

}  // namespace nb
