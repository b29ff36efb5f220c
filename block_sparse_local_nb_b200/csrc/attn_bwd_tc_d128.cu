// Banded block-sparse local attention backward, main kernel for d = 128, on
// the 5th-generation tensor cores (tcgen05 + TMEM), bf16 in / fp32 accumulate.
// (NucleoByte page, section 3 "Custom Backpropagation": P recomputed from the
// stored log-sum-exp, D_i = sum_k dO_ik O_ik, dS = P (dP - D); gradients of
// shared key/value blocks accumulated with atomic adds.)
//
// Work item = one key tile of 128 keys of one (batch, head), as for d = 64
// (attn_bwd_tc.cu), but the item's query blocks [4t - R, 4t + 3 + R] (causal:
// [4t, 4t + 3 + R]) are taken in chunks of 64 queries.  At d = 128 a 128-query
// chunk of Q and dO is 64 KB, which leaves room for one stage only, and the
// whole chunk pipeline (load, S/dP, softmax arithmetic, gradient products)
// then runs in series; 64-query chunks fit three stages, Pᵀ in TMEM, and
// every product keeps M = 128:
//   Sᵀ  = K Qᵀ          dPᵀ = V dOᵀ                 (M 128 keys, N 64, K d)
//   Pᵀ  = 2^(Sᵀ scale log2e - lse log2e),  dSᵀ = Pᵀ (dPᵀ - D)   (CUDA cores)
//   dV += Pᵀ dO         dK += dSᵀ Q                 (M 128 keys, N d, K 64)
//   dQ_cᵀ = Kᵀ dSᵀ                                  (M d, N 64, K 128 keys)
// dK and dV accumulate in TMEM over the item's chunks (deterministic); dQ_c is
// computed transposed (d on the TMEM lanes) and added into the fp32
// accumulator in global memory with TMA bulk reduce-adds.
//
// TMEM (512 columns): Sᵀ [0, 64), dPᵀ [64, 128), Pᵀ as bf16 pairs [128, 160),
// dQ_cᵀ [192, 256), dV [256, 384), dK [384, 512).
// Shared memory: K and V tiles (64 KB), three Q/dO stages (96 KB), dSᵀ
// (16 KB), four dQ staging boxes (32 KB).
//
// Warp roles (512 threads, four warpgroups with reallocated registers):
// warpgroup 0: warp 0 TMA producer, warp 1 TMEM owner and S/dP issuer, warp 2
// issuer of the dV/dK/dQ products, warp 3 the dK/dV tile stores; warpgroups
// 1-2: gradient warps (thread = key row; half hf owns the chunk's query block
// hf, 32 queries); warpgroup 3: dQ warps (thread = one of the d columns),
// each warp staging and reducing its own 32-column box.  All waits are
// bounded (see sm100.cuh).
#include <math.h>

#include "nb_internal.h"
#include "schedule.cuh"
#include "sm100.cuh"

namespace nb {
namespace {

using namespace sm100;

constexpr int D = 128;
constexpr int kThreads = 512;
constexpr int kLaunchRegs = 65536 / kThreads / 8 * 8;  // per thread at launch
constexpr int kKeys = 128;  // keys per item
constexpr int kQ = 64;      // queries per chunk (two query blocks)
constexpr int kNS = 3;      // Q/dO stages
constexpr int kTile = kKeys * D * 2;   // one [128 x 128] bf16 tile (two 16 KB slabs)
constexpr int kSlab = kKeys * 128;     // one 128-row x 128-byte swizzled slab
constexpr int kQTile = kQ * D * 2;     // one [64 x 128] bf16 chunk (two 8 KB slabs)
constexpr int kQSlab = kQ * 128;
constexpr float kLog2e = 1.4426950408889634f;

// shared memory
constexpr int oK = 0;                      // K tile, V tile after it
constexpr int oQ = 2 * kTile;              // stage s: Q at oQ + 2 s kQTile, dO after it
constexpr int oDS = oQ + kNS * 2 * kQTile; // dSᵀ: 128 keys x 64 queries bf16 (one slab)
constexpr int oStg = oDS + kSlab;          // dQ staging: box w (64 rows x 32 fp32) at oStg + w 8 KB
constexpr int kStgBox = kQ * 128;
constexpr int oLD = oStg + 4 * kStgBox;    // stage s: -lse log2e [64], D [64]
constexpr int oBar = oLD + kNS * 512;
constexpr int bKVFull = 0, bKVFree = 1, bQDFull = 2, bQDFree = bQDFull + kNS,
              bSDPFull = bQDFree + kNS, bSDPFree = bSDPFull + 1, bPDSFull = bSDPFree + 1,
              bPDSFree = bPDSFull + 1, bDQFull = bPDSFree + 1, bDQFree = bDQFull + 1,
              bDKVFull = bDQFree + 1, bDKVFree = bDKVFull + 1, bOutFull = bDKVFree + 1,
              bDone = bOutFull + 1, nBar = bDone + 1;
constexpr int oSlot = oBar + nBar * 8;
constexpr int oSched = oSlot + 16;  // work-order prefix table
constexpr int kSmem = oSched + kSchedBytes + 1024;
static_assert(kSmem <= 227 * 1024, "shared memory per CTA");

// tensor memory
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t tS = 0, tDP = 64, tP = 128, tDQ = 192, tDV = 256, tDK = 384;

// registers per thread after reallocation: control warpgroup, each gradient
// warpgroup, dQ warpgroup
constexpr int kRegsCtl = 48, kRegsGrad = 168, kRegsDq = 128;
static_assert(128 * (kRegsCtl + 2 * kRegsGrad + kRegsDq) <= 65536, "register budget");

struct Params {
  AttnArgs a;
  BwdWorkspace ws;
  int ntiles;  // key tiles per (batch, head)
  int items;
};

struct Item {
  int b, h, tile, L, I0, nch;
};

__device__ __forceinline__ Item decode_bht(const Params& p, int b, int h, int tile, int L) {
  const AttnArgs& a = p.a;
  Item x;
  x.b = b;
  x.h = h;
  x.tile = tile;
  x.L = L;  // clamped to [0, n]
  const int nb = a.n / kBlock;
  x.I0 = 0;
  x.nch = 0;
  if (x.tile * kKeys < x.L) {
    const int kb_last = min(x.tile * 4 + 3, nb - 1);
    x.I0 = a.causal ? x.tile * 4 : max(0, x.tile * 4 - a.R);
    const int I1 = min(min(kb_last + a.R, nb - 1), (x.L - 1) / kBlock);
    x.nch = (I1 - x.I0 + 2) / 2;  // two query blocks per chunk
  }
  return x;
}

__device__ __forceinline__ Item decode(const Params& p, int it) {
  const int bh = it / p.ntiles;
  const int b = bh / p.a.heads;
  const int L = p.a.lengths ? p.a.lengths[b] : p.a.n;
  return decode_bht(p, b, bh - b * p.a.heads, it - bh * p.ntiles, min(max(L, 0), p.a.n));
}

__device__ __forceinline__ Item sched_item(const Params& p, const Sched& s, int k) {
  if (!s.balanced) return decode(p, k);
  int b, h, tile;
  sched_nonempty(s, p.a.batch, p.a.heads, k, b, h, tile);
  return decode_bht(p, b, h, tile, sched_length(s, p.a, b));
}

enum : int { kErrKVFree = 0x51, kErrQDFree, kErrKVFull, kErrQDFull, kErrSDPFree, kErrDQFree,
             kErrPDSFull, kErrDKVFree, kErrGQD, kErrSDPFull, kErrPDSFree, kErrDKVFull,
             kErrDQFull, kErrDone, kErrOutFull };

__device__ int producer(const Params& p, const Sched& sch, uint32_t base, const CUtensorMap* tk,
                        const CUtensorMap* tv, const CUtensorMap* tq, const CUtensorMap* tdo) {
  const AttnArgs& a = p.a;
  const uint32_t bar = base + oBar;
  int g = 0, tc = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    if (x.nch == 0) continue;
    const int bh = x.b * a.heads + x.h;
    if (!mbar_wait(bar + 8 * bKVFree, (tc & 1) ^ 1)) return kErrKVFree;
    mbar_arrive_expect_tx(bar + 8 * bKVFull, 2 * kTile);
#pragma unroll
    for (int s = 0; s < D / 64; ++s) {
      tma_load_3d(base + oK + s * kSlab, tk, bar + 8 * bKVFull, s * 64, x.tile * kKeys, bh);
      tma_load_3d(base + oK + kTile + s * kSlab, tv, bar + 8 * bKVFull, s * 64, x.tile * kKeys, bh);
    }
    for (int c = 0; c < x.nch; ++c) {
      const int G = g + c, st = G % kNS;
      if (!mbar_wait(bar + 8 * (bQDFree + st), ((G / kNS) & 1) ^ 1)) return kErrQDFree;
      const int q0 = (x.I0 + 2 * c) * kBlock;
      const int rows = min(kQ, a.n - q0);  // lse / D rows that exist
      const uint32_t full = bar + 8 * (bQDFull + st);
      mbar_arrive_expect_tx(full, 2 * kQTile + 8 * rows);
      const uint32_t sq = base + oQ + st * 2 * kQTile;
#pragma unroll
      for (int s = 0; s < D / 64; ++s) {
        tma_load_3d(sq + s * kQSlab, tq, full, s * 64, q0, bh);
        tma_load_3d(sq + kQTile + s * kQSlab, tdo, full, s * 64, q0, bh);
      }
      const int64_t row0 = static_cast<int64_t>(bh) * a.n + q0;
      const uint32_t sld = base + oLD + st * 512;
      bulk_load(sld, p.ws.nlse2 + row0, 4 * rows, full);
      bulk_load(sld + 256, p.ws.D + row0, 4 * rows, full);
    }
    g += x.nch;
    ++tc;
  }
  return 0;
}

// Sᵀ = K Qᵀ and dPᵀ = V dOᵀ for every chunk (warp 1, one thread); chunk G + 1
// goes in as soon as the gradient warps hold chunk G's values in registers.
__device__ int sdp_issuer(const Params& p, const Sched& sch, uint32_t base, uint32_t tmem) {
  const uint32_t bar = base + oBar;
  constexpr uint32_t kIdS = idesc_bf16_f32(128, kQ, false, false);  // both K-major
  const uint64_t dK = smem_desc_sw128(base + oK, 0, 1024);
  const uint64_t dV = smem_desc_sw128(base + oK + kTile, 0, 1024);
  int g = 0, tc = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    if (x.nch == 0) continue;
    if (!mbar_wait(bar + 8 * bKVFull, tc & 1)) return kErrKVFull;
    for (int c = 0; c < x.nch; ++c) {
      const int G = g + c, st = G % kNS;
      const uint32_t sQ = base + oQ + st * 2 * kQTile;
      const uint64_t dQ = smem_desc_sw128(sQ, 0, 1024), ddO = smem_desc_sw128(sQ + kQTile, 0, 1024);
      if (!mbar_wait(bar + 8 * (bQDFull + st), (G / kNS) & 1)) return kErrQDFull;
      if (!mbar_wait(bar + 8 * bSDPFree, (G & 1) ^ 1)) return kErrSDPFree;
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t oa = ((k >> 2) * kSlab + (k & 3) * 32) >> 4;   // descriptor units
        const uint32_t ob = ((k >> 2) * kQSlab + (k & 3) * 32) >> 4;
        mma_bf16_ss(tmem + tS, desc_add(dK, oa), desc_add(dQ, ob), kIdS, k > 0);
        mma_bf16_ss(tmem + tDP, desc_add(dV, oa), desc_add(ddO, ob), kIdS, k > 0);
      }
      mma_commit(bar + 8 * bSDPFull);
    }
    g += x.nch;
    ++tc;
  }
  return 0;
}

// dV += Pᵀ dO, dK += dSᵀ Q and dQ_cᵀ = Kᵀ dSᵀ for every chunk (warp 2, one
// thread).  The S/dP products of a chunk completed before its gradient warps
// began, so a commit here also covers every read of that chunk's Q/dO.
__device__ int grad_issuer(const Params& p, const Sched& sch, uint32_t base, uint32_t tmem) {
  const uint32_t bar = base + oBar;
  constexpr uint32_t kIdKV = idesc_bf16_f32(128, D, false, true);  // Pᵀ dO, dSᵀ Q
  constexpr uint32_t kIdQ = idesc_bf16_f32(128, kQ, true, true);   // Kᵀ dSᵀ
  const uint64_t dSk = smem_desc_sw128(base + oDS, 0, 1024);       // dSᵀ as a K-major A
  const uint64_t dSm = smem_desc_sw128(base + oDS, kSlab, 1024);   // dSᵀ as an MN-major B
  const uint64_t dKm = smem_desc_sw128(base + oK, kSlab, 1024);    // Kᵀ as an MN-major A
  int g = 0, tc = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    if (x.nch == 0) continue;
    for (int c = 0; c < x.nch; ++c) {
      const int G = g + c, st = G % kNS;
      const uint32_t sQ = base + oQ + st * 2 * kQTile;
      const uint64_t dQm = smem_desc_sw128(sQ, kQSlab, 1024);
      const uint64_t ddOm = smem_desc_sw128(sQ + kQTile, kQSlab, 1024);
      const bool acc = c > 0;
      if (!mbar_wait(bar + 8 * bPDSFull, G & 1)) return kErrPDSFull;
      if (c == 0 && !mbar_wait(bar + 8 * bDKVFree, (tc & 1) ^ 1)) return kErrDKVFree;
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < kQ / 16; ++k) {  // k over the chunk's queries
        const uint32_t mn = (k * 2048) >> 4;  // 16 rows of an MN-major operand
        mma_bf16_ts(tmem + tDV, tmem + tP + 8 * k, desc_add(ddOm, mn), kIdKV, acc || k > 0);
        mma_bf16_ss(tmem + tDK, desc_add(dSk, (k * 32) >> 4), desc_add(dQm, mn), kIdKV,
                    acc || k > 0);
      }
      // Q and dO are last read by the products above
      mma_commit(bar + 8 * (bQDFree + st));
      if (!mbar_wait(bar + 8 * bDQFree, (G & 1) ^ 1)) return kErrDQFree;
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < kKeys / 16; ++k) {  // k over the tile's keys
        const uint32_t mn = (k * 2048) >> 4;
        mma_bf16_ss(tmem + tDQ, desc_add(dKm, mn), desc_add(dSm, mn), kIdQ, k > 0);
      }
      mma_commit(bar + 8 * bPDSFree);
      mma_commit(bar + 8 * bDQFull);
      if (c == x.nch - 1) mma_commit(bar + 8 * bDKVFull);
    }
    g += x.nch;
    ++tc;
  }
  return 0;
}

// dK/dV tile stores (warp 3, one thread): the gradient warps stage an item's dK
// and dV in its K and V buffers (free once its last products, the dQ product
// reading K included, have completed); the buffer goes back to the producer
// once the stores have read it.
__device__ int out_storer(const Params& p, const Sched& sch, uint32_t base, const CUtensorMap* tdk,
                          const CUtensorMap* tdv) {
  const uint32_t bar = base + oBar;
  int tc = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    if (x.nch == 0) continue;
    const int bh = x.b * p.a.heads + x.h;
    if (!mbar_wait(bar + 8 * bOutFull, tc & 1)) return kErrOutFull;
#pragma unroll
    for (int s = 0; s < D / 64; ++s) {
      tma_store_3d(tdk, base + oK + s * kSlab, s * 64, x.tile * kKeys, bh);
      tma_store_3d(tdv, base + oK + kTile + s * kSlab, s * 64, x.tile * kKeys, bh);
    }
    bulk_commit();
    bulk_wait_read0();
    mbar_arrive(bar + 8 * bKVFree);
    ++tc;
  }
  bulk_wait_all0();  // the stores have landed before the CTA exits
  return 0;
}

// Gradient warps: thread = key row r; half hf owns query block hf of the
// chunk (queries [32 hf, 32 hf + 32)).
template <bool kCausal>
__device__ int grad_warps(const Params& p, const Sched& sch, uint32_t base, uint8_t* gbase,
                          uint32_t tmem, int wq, int hf, int lane) {
  const AttnArgs& a = p.a;
  const uint32_t bar = base + oBar;
  const int r = wq * 32 + lane;
  const uint32_t trow = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  const int nb = a.n / kBlock;
  const float sl2 = a.scale * kLog2e;
  auto all_ok = [](bool ok) { return __all_sync(0xffffffffu, ok); };
  // a key tile entirely past its sequence's length: dK = dV = 0 (first group dK, second dV)
  auto zero_tile = [&](const Item& x) {
    const int64_t row0 = (static_cast<int64_t>(x.b) * a.heads + x.h) * a.n + x.tile * kKeys;
    const int rows = min(kKeys, a.n - x.tile * kKeys);
    uint4* out = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(hf == 0 ? a.dk : a.dv) +
                                          row0 * D);
    for (int i = r; i < rows * (D / 8); i += 128) out[i] = make_uint4(0, 0, 0, 0);
  };
  int g = 0, tc = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    const int k = x.tile * kKeys + r;
    if (x.nch == 0) {  // every key of the tile is padding
      zero_tile(x);
      continue;
    }
    const bool row_valid = k < x.L;
    const int kb = k / kBlock;
    for (int c = 0; c < x.nch; ++c) {
      const int G = g + c, st = G % kNS;
      if (!all_ok(mbar_wait(bar + 8 * (bQDFull + st), (G / kNS) & 1))) return kErrGQD;
      if (!all_ok(mbar_wait(bar + 8 * bSDPFull, G & 1))) return kErrSDPFull;
      tc_fence_after();
      const float* nl = reinterpret_cast<const float*>(gbase + oLD + st * 512) + 32 * hf;
      const float* Dv = nl + 64;
      float sv[32], dpv[32];
      tmem_ld32(trow + tS + 32 * hf, sv);
      tmem_ld32(trow + tDP + 32 * hf, dpv);
      tmem_wait_ld();
      reg_fence(sv);
      reg_fence(dpv);
      tc_fence_before();  // S and dP of this chunk are in registers: TMEM may be reused
      mbar_arrive(bar + 8 * bSDPFree);
      const int qb = x.I0 + 2 * c + hf;  // this half's query block
      const bool vis = row_valid && qb < nb &&
                       (kCausal ? (qb >= kb && qb - kb <= a.R) : abs(qb - kb) <= a.R);
      // causal, diagonal block: queries before this key (index < k mod 32) see it not
      const int cut = kCausal && qb == kb ? (k & (kBlock - 1)) : 0;
      uint32_t wp[16], ws[16];  // packed bf16 Pᵀ and dSᵀ for this thread's 32 queries
      if (vis) {
        const float2 sl = make_float2(sl2, sl2);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const float4 n0 = *reinterpret_cast<const float4*>(nl + 8 * cc);
          const float4 n1 = *reinterpret_cast<const float4*>(nl + 8 * cc + 4);
          const float4 d0 = *reinterpret_cast<const float4*>(Dv + 8 * cc);
          const float4 d1 = *reinterpret_cast<const float4*>(Dv + 8 * cc + 4);
          const float2 nv[4] = {make_float2(n0.x, n0.y), make_float2(n0.z, n0.w),
                                make_float2(n1.x, n1.y), make_float2(n1.z, n1.w)};
          const float2 nd[4] = {make_float2(d0.x, d0.y), make_float2(d0.z, d0.w),
                                make_float2(d1.x, d1.y), make_float2(d1.z, d1.w)};
#pragma unroll
          for (int e = 0; e < 4; ++e) {  // pairs of queries, packed fp32x2 arithmetic
            const int i = 8 * cc + 2 * e;
            float2 xv = __ffma2_rn(make_float2(sv[i], sv[i + 1]), sl, nv[e]);  // -inf: padding
            if (i < cut) xv.x = -INFINITY;
            if (i + 1 < cut) xv.y = -INFINITY;
            const float2 pe = make_float2(ex2_approx(xv.x), ex2_approx(xv.y));
            const float2 de = __fmul2_rn(pe, __fadd2_rn(make_float2(dpv[i], dpv[i + 1]), nd[e]));
            wp[4 * cc + e] = pack_bf16(pe.x, pe.y);
            ws[4 * cc + e] = pack_bf16(de.x, de.y);
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) wp[e] = ws[e] = 0u;
      }
      // the previous chunk's products must be done reading Pᵀ and dSᵀ
      if (!all_ok(mbar_wait(bar + 8 * bPDSFree, (G & 1) ^ 1))) return kErrPDSFree;
      tmem_st16u(trow + tP + 16 * hf, wp);
      uint8_t* srow = gbase + oDS + r * 128;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
        *reinterpret_cast<uint4*>(srow + (((4 * hf + cc) ^ (r & 7)) << 4)) =
            make_uint4(ws[4 * cc], ws[4 * cc + 1], ws[4 * cc + 2], ws[4 * cc + 3]);
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar + 8 * bPDSFull);
    }
    // epilogue: this thread's row of dK (first half, times 1/sqrt(d)) or dV
    // (second half) as bf16 into the item's K (dK) or V (dV) buffer, as 128-byte
    // swizzled slabs for the tile stores
    if (!all_ok(mbar_wait(bar + 8 * bDKVFull, tc & 1))) return kErrDKVFull;
    tc_fence_after();
    uint32_t outp[D / 2];
    const float mul = row_valid ? (hf == 0 ? a.scale : 1.f) : 0.f;
    const uint32_t tsrc = trow + (hf == 0 ? tDK : tDV);
#pragma unroll
    for (int j = 0; j < D / 32; ++j) {
      float v[32];
      tmem_ld32(tsrc + 32 * j, v);
      tmem_wait_ld();
      reg_fence(v);
#pragma unroll
      for (int i = 0; i < 16; ++i) outp[16 * j + i] = pack_bf16(v[2 * i] * mul, v[2 * i + 1] * mul);
    }
    tc_fence_before();
    mbar_arrive(bar + 8 * bDKVFree);
    uint8_t* stg = gbase + oK + hf * kTile + r * 128;
#pragma unroll
    for (int gc = 0; gc < D / 8; ++gc)  // 16-byte chunk of the output row
      *reinterpret_cast<uint4*>(stg + (gc >> 3) * kSlab + (((gc & 7) ^ (r & 7)) << 4)) =
          make_uint4(outp[4 * gc], outp[4 * gc + 1], outp[4 * gc + 2], outp[4 * gc + 3]);
    fence_proxy_async_smem();
    mbar_arrive(bar + 8 * bOutFull);
    g += x.nch;
    ++tc;
  }
  if (sch.balanced) {  // second pass: the empty tiles, listed directly
    for (int e = blockIdx.x; e < p.items - sch.count; e += gridDim.x) {
      int b, h, tile;
      sched_empty(sch, a.batch, a.heads, p.ntiles, e, b, h, tile);
      zero_tile(decode_bht(p, b, h, tile, sched_length(sch, a, b)));
    }
  }
  return 0;
}

// dQ warps: thread = column d of dQ (TMEM lane d of dQ_cᵀ).  Warp w owns
// columns [32 w, 32 w + 32): it writes them for the chunk's 64 queries into
// its own staging box and one lane reduces the box into the accumulator.
__device__ int dq_warps(const Params& p, const Sched& sch, uint32_t base, uint8_t* gbase,
                        uint32_t tmem, int wq, int lane, const CUtensorMap* tdq) {
  const AttnArgs& a = p.a;
  const uint32_t bar = base + oBar;
  const uint32_t trow = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  auto all_ok = [](bool ok) { return __all_sync(0xffffffffu, ok); };
  uint8_t* box = gbase + oStg + wq * kStgBox;
  int g = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    if (x.nch == 0) continue;
    const int bh = x.b * a.heads + x.h;
    for (int c = 0; c < x.nch; ++c) {
      const int G = g + c;
      const int q0 = (x.I0 + 2 * c) * kBlock;
      if (!all_ok(mbar_wait(bar + 8 * bDQFull, G & 1))) return kErrDQFull;
      tc_fence_after();
      float v[2][32];  // this column's values for the chunk's 64 queries
      tmem_ld32(trow + tDQ, v[0]);
      tmem_ld32(trow + tDQ + 32, v[1]);
      tmem_wait_ld();
      reg_fence(v[0]);
      reg_fence(v[1]);
      tc_fence_before();
      mbar_arrive(bar + 8 * bDQFree);
      if (lane == 0) bulk_wait_read0();  // the previous reduce-add has read the box
      __syncwarp();
      // box: 64 rows (queries) x 32 fp32 (this warp's columns), 128-byte swizzle
#pragma unroll
      for (int q = 0; q < kQ; ++q)
        *reinterpret_cast<float*>(box + q * 128 + ((((lane >> 2) ^ (q & 7))) << 4) +
                                  (lane & 3) * 4) = v[q >> 5][q & 31];
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_reduce_add_3d(tdq, base + oStg + wq * kStgBox, 32 * wq, q0, bh);
        bulk_commit();
      }
    }
    g += x.nch;
  }
  if (lane == 0) bulk_wait_all0();  // the last reduce-adds have read shared memory and landed
  return 0;
}

template <bool kCausal>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_tc_d128_kernel(const __grid_constant__ CUtensorMap tk,
                            const __grid_constant__ CUtensorMap tv,
                            const __grid_constant__ CUtensorMap tq,
                            const __grid_constant__ CUtensorMap tdo,
                            const __grid_constant__ CUtensorMap tdq,
                            const __grid_constant__ CUtensorMap tdk,
                            const __grid_constant__ CUtensorMap tdv, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bar = base + oBar;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar + 8 * bKVFull, 1);
    mbar_init(bar + 8 * bKVFree, 1);
    for (int i = 0; i < kNS; ++i) {
      mbar_init(bar + 8 * (bQDFull + i), 1);
      mbar_init(bar + 8 * (bQDFree + i), 1);
    }
    mbar_init(bar + 8 * bSDPFull, 1);
    mbar_init(bar + 8 * bSDPFree, 256);
    mbar_init(bar + 8 * bPDSFull, 256);
    mbar_init(bar + 8 * bPDSFree, 1);
    mbar_init(bar + 8 * bDQFull, 1);
    mbar_init(bar + 8 * bDQFree, 128);
    mbar_init(bar + 8 * bDKVFull, 1);
    mbar_init(bar + 8 * bDKVFree, 256);
    mbar_init(bar + 8 * bOutFull, 256);
    mbar_init(bar + 8 * bDone, 2);  // one commit per MMA-issuing thread
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tk);
    prefetch_tmap(&tv);
    prefetch_tmap(&tq);
    prefetch_tmap(&tdo);
    prefetch_tmap(&tdq);
    prefetch_tmap(&tdk);
    prefetch_tmap(&tdv);
  }
  if (warp == 1) {
    tmem_alloc(base + oSlot, kTmemCols);
    tmem_relinquish();
  }
  pdl_wait();  // everything above overlaps the previous kernel's tail
  if (warp == 0) sched_build(reinterpret_cast<int*>(gbase + oSched), p.a, kKeys, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + oSlot);
  const Sched sch = sched_view(reinterpret_cast<const int*>(gbase + oSched), p.a, p.items);

  // Role branches never join again: each ends with the CTA barrier, after which
  // warp 1 waits for the tensor cores and frees the TMEM.
  if (warp < 4) {
    regs_dec<kRegsCtl, kLaunchRegs>();
    int err = 0;
    if (warp == 0 && lane == 0) err = producer(p, sch, base, &tk, &tv, &tq, &tdo);
    if (warp == 1 && lane == 0) err = sdp_issuer(p, sch, base, tmem);
    if (warp == 2 && lane == 0) err = grad_issuer(p, sch, base, tmem);
    if (warp == 3 && lane == 0) err = out_storer(p, sch, base, &tdk, &tdv);
    if (err) record_error(p.a.err, err);
    pdl_trigger();  // this CTA's work is issued: the next kernel may start launching
    __syncthreads();
    if (warp == 2 && lane == 0) mma_commit(bar + 8 * bDone);
    if (warp == 1) {
      if (lane == 0) {
        mma_commit(bar + 8 * bDone);
        if (!mbar_wait(bar + 8 * bDone, 0)) record_error(p.a.err, kErrDone);
      }
      __syncwarp();
      tc_fence_after();
      tmem_dealloc(tmem, kTmemCols);
    }
  } else if (warp < 12) {
    regs_inc<kRegsGrad, kLaunchRegs>();
    const int err = grad_warps<kCausal>(p, sch, base, gbase, tmem, warp & 3, (warp - 4) >> 2, lane);
    if (err) record_error(p.a.err, err);
    pdl_trigger();
    __syncthreads();
  } else {
    regs_dec<kRegsDq, kLaunchRegs>();
    const int err = dq_warps(p, sch, base, gbase, tmem, warp & 3, lane, &tdq);
    if (err) record_error(p.a.err, err);
    pdl_trigger();
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_bwd_main_tc_d128(const AttnArgs& a, int64_t rows, cudaStream_t stream) {
  const int64_t heads_total = static_cast<int64_t>(a.batch) * a.heads;
  Params p;
  p.a = a;
  p.ws = bwd_workspace(a.workspace, rows);
  CUtensorMap tk, tv, tq, tdo, tdq, tdk, tdv;
  if (!make_tmap_bf16_rows(&tk, a.k, D, a.n, heads_total, kKeys) ||
      !make_tmap_bf16_rows(&tv, a.v, D, a.n, heads_total, kKeys) ||
      !make_tmap_bf16_rows(&tq, a.q, D, a.n, heads_total, kQ) ||
      !make_tmap_bf16_rows(&tdo, a.dout, D, a.n, heads_total, kQ) ||
      !make_tmap_rows(&tdq, p.ws.dqacc, true, D, a.n, heads_total, 32, kQ) ||
      !make_tmap_bf16_rows(&tdk, a.dk, D, a.n, heads_total, kKeys) ||
      !make_tmap_bf16_rows(&tdv, a.dv, D, a.n, heads_total, kKeys))
    return cudaErrorInvalidValue;
  p.ntiles = (a.n + kKeys - 1) / kKeys;
  const int64_t items = heads_total * p.ntiles;
  if (items > (1ll << 30)) return cudaErrorInvalidValue;
  p.items = static_cast<int>(items);
  auto kernel = a.causal ? attn_bwd_tc_d128_kernel<true> : attn_bwd_tc_d128_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(items < num_sms() ? items : num_sms());
  return launch_pdl(kernel, dim3(grid), dim3(kThreads), kSmem, stream, tk, tv, tq, tdo, tdq, tdk,
                    tdv, p);
}

}  // namespace nb
