// Banded block-sparse local attention backward, main kernel for d = 64 (d = 128
// is attn_bwd_tc_d128.cu), on the 5th-generation tensor cores (tcgen05 +
// TMEM), bf16 in / fp32 accumulate.
// (NucleoByte page, section 3 "Custom Backpropagation": P recomputed from the
// stored log-sum-exp, D_i = sum_k dO_ik O_ik, dS = P (dO V^T - D); gradients of
// shared key/value blocks accumulated with atomic adds.)
//
// Work item = one key tile of 128 keys (four key blocks) of one (batch, head).
// (The causal band, the kCausal instantiation, takes query blocks 4t ..
// 4t + 3 + R and zeroes P for queries before their key in the diagonal block.)
// The band is symmetric, so its dK and dV need only the query blocks
// [4t - R, 4t + 3 + R], taken in chunks of 128 queries.  Per chunk, with keys
// on the TMEM lanes (M = 128):
//   S^T  = K Q^T          dP^T = V dO^T                       (N 128, K d)
//   P^T  = 2^(S^T scale log2e - lse log2e),  dS^T = P^T (dP^T - D)   (CUDA cores,
//          packed fp32x2 arithmetic)
//   dV  += P^T dO         dK  += dS^T Q                        (N d, K 128)
//   dQ_c = dS K           (queries on the lanes: dS^T read as an MN-major A)
// dK and dV accumulate in TMEM over the item's chunks (deterministic); dQ_c is
// added into an fp32 accumulator in global memory with a TMA bulk reduce-add.
//
// Warp roles (512 threads, four warpgroups with reallocated registers):
// warpgroup 0: warp 0 TMA producer (K, V tiles; Q, dO chunks; the chunk's lse
// and D rows by bulk copy), warp 1 TMEM owner and S/dP issuer, warp 2 issuer of
// the dV/dK/dQ products (two issuing threads, so neither stream of MMAs waits
// behind the other's barriers), warp 3 the dK/dV tile stores; warpgroups 1-2:
// gradient warps, one warpgroup per half of the chunk's query columns, thread =
// key row; they also stage dK (first) and dV (second) of an item in its K/V
// buffer after the next item's first chunk (so the wait for the item's last
// products overlaps that chunk's arithmetic);
// warpgroup 3: dQ warps, thread = query row; each warp stages its 32 rows of
// dQ_c in its own shared-memory box and reduce-adds them into global memory.
// All waits are bounded (see sm100.cuh).
#include <math.h>

#include "nb_internal.h"
#include "schedule.cuh"
#include "sm100.cuh"

namespace nb {
namespace {

using namespace sm100;

constexpr int kThreads = 512;
constexpr int kLaunchRegs = 65536 / kThreads / 8 * 8;  // per thread at launch

constexpr int kRows = 128;        // keys per item, queries per chunk
constexpr int kSlab = 128 * 128;  // one swizzled box: 128 rows x 128 bytes
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Cfg {
  static_assert(D == 64, "this kernel is the d = 64 one");
  // K/V tiles double-buffered, three Q/dO stages; P^T kept in TMEM (64 spare
  // columns) as the A operand of dV; dQ staged through one 128 x 32 fp32 area
  // (a 32 x 32 box per dQ warp),
  // so a chunk's Q/dO buffer is free as soon as its gradient products complete.
  static constexpr int NKV = 2;  // K/V tile buffers
  static constexpr int NS = 3;   // Q/dO chunk stages
  static constexpr int kTile = kRows * D * 2;  // one [128 x D] bf16 tile
  static constexpr int kPT = kRows * kRows * 2;  // one [128 x 128] bf16 tile
  static constexpr int oK = 0;                   // buffer i: K at oK + 2 i kTile, V after it
  static constexpr int oQ = NKV * 2 * kTile;     // stage s: Q at oQ + 2 s kTile, dO after it
  static constexpr int oDS = oQ + NS * 2 * kTile;  // dS^T tile
  static constexpr int oStg = oDS + kPT;  // dQ staging: warp w's 32 x 32 fp32 box at + 4 KB w
  // The dK/dV epilogue of an item is deferred past the next item's first
  // chunk (the next item's K/V tile has a buffer of its own).
  static constexpr int oLD = oStg + kSlab;  // stage s: -lse log2e, D
  static constexpr int oBar = oLD + NS * 1024;
  static constexpr int bKVFull = 0, bKVFree = bKVFull + NKV, bQDFull = bKVFree + NKV,
                       bQDFree = bQDFull + NS, bSDPFull = bQDFree + NS, bSDPFree = bSDPFull + 1,
                       bPDSFull = bSDPFree + 1, bPDSFree = bPDSFull + 1, bDQFull = bPDSFree + 1,
                       bDQFree = bDQFull + 1, bDKVFull = bDQFree + 1, bDKVFree = bDKVFull + 1,
                       bOutFull = bDKVFree + 1,
                       bDone = bOutFull + NKV,
                       nBar = bDone + 1;
  static constexpr int oSlot = oBar + nBar * 8;
  static constexpr int oSched = oSlot + 16;  // work-order prefix table
  static constexpr int kSmem = oSched + kSchedBytes + 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t tS = 0, tDP = 128, tDV = 256, tDK = 256 + D, tDQ = 384;
  static constexpr uint32_t tP = 448;                 // P^T, bf16 pairs
  // registers per thread after reallocation: TMA/MMA warpgroup, each gradient
  // warpgroup, dQ warpgroup (the 16 warps share the 64K-register file)
  static constexpr int kRegsCtl = 64;
  static constexpr int kRegsGrad = 176;
  static constexpr int kRegsDq = 96;
  static_assert(128 * (kRegsCtl + 2 * kRegsGrad + kRegsDq) <= 65536, "register budget");
};

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
  if (x.tile * kRows < x.L) {
    const int kb_last = min(x.tile * 4 + 3, nb - 1);
    x.I0 = a.causal ? x.tile * 4 : max(0, x.tile * 4 - a.R);  // causal: queries at or after the keys
    const int I1 = min(min(kb_last + a.R, nb - 1), (x.L - 1) / kBlock);
    x.nch = (I1 - x.I0 + 4) / 4;
  }
  return x;
}

// Item `it` of the round-robin order over every tile.
__device__ __forceinline__ Item decode(const Params& p, int it) {
  const int bh = it / p.ntiles;
  const int b = bh / p.a.heads;
  const int L = p.a.lengths ? p.a.lengths[b] : p.a.n;
  return decode_bht(p, b, bh - b * p.a.heads, it - bh * p.ntiles, min(max(L, 0), p.a.n));
}

// Item k of the first pass (non-empty tiles when balanced, else every tile).
__device__ __forceinline__ Item sched_item(const Params& p, const Sched& s, int k) {
  if (!s.balanced) return decode(p, k);
  int b, h, tile;
  sched_nonempty(s, p.a.batch, p.a.heads, k, b, h, tile);
  return decode_bht(p, b, h, tile, sched_length(s, p.a, b));
}

enum : int { kErrKVFree = 0x31, kErrQDFree, kErrKVFull, kErrQDFull, kErrSDPFree, kErrDQFree,
             kErrPDSFull, kErrDKVFree, kErrGQD, kErrSDPFull, kErrPDSFree, kErrDKVFull,
             kErrDQFull, kErrDone, kErrOutFull };

template <int D>
__device__ int producer(const Params& p, const Sched& sch, uint32_t base, const CUtensorMap* tk,
                        const CUtensorMap* tv, const CUtensorMap* tq, const CUtensorMap* tdo) {
  using C = Cfg<D>;
  const AttnArgs& a = p.a;
  const uint32_t bar = base + C::oBar;
  int g = 0, tc = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    if (x.nch == 0) continue;
    const int bh = x.b * a.heads + x.h;
    const int kvb = tc % C::NKV;
    const uint32_t kvfull = bar + 8 * (C::bKVFull + kvb);
    if (!mbar_wait(bar + 8 * (C::bKVFree + kvb), ((tc / C::NKV) & 1) ^ 1)) return kErrKVFree;
    mbar_arrive_expect_tx(kvfull, 2 * C::kTile);
    const uint32_t sk = base + C::oK + kvb * 2 * C::kTile;
#pragma unroll
    for (int s = 0; s < D / 64; ++s) {
      tma_load_3d(sk + s * kSlab, tk, kvfull, s * 64, x.tile * kRows, bh);
      tma_load_3d(sk + C::kTile + s * kSlab, tv, kvfull, s * 64, x.tile * kRows, bh);
    }
    for (int c = 0; c < x.nch; ++c) {
      const int G = g + c, st = G % C::NS;
      if (!mbar_wait(bar + 8 * (C::bQDFree + st), ((G / C::NS) & 1) ^ 1)) return kErrQDFree;
      const int q0 = (x.I0 + 4 * c) * kBlock;
      const int rows = min(kRows, a.n - q0);  // lse / D rows that exist
      const uint32_t full = bar + 8 * (C::bQDFull + st);
      mbar_arrive_expect_tx(full, 2 * C::kTile + 8 * rows);
      const uint32_t sq = base + C::oQ + st * 2 * C::kTile;
#pragma unroll
      for (int s = 0; s < D / 64; ++s) {
        tma_load_3d(sq + s * kSlab, tq, full, s * 64, q0, bh);
        tma_load_3d(sq + C::kTile + s * kSlab, tdo, full, s * 64, q0, bh);
      }
      const int64_t row0 = static_cast<int64_t>(bh) * a.n + q0;
      const uint32_t sld = base + C::oLD + st * 1024;
      bulk_load(sld, p.ws.nlse2 + row0, 4 * rows, full);
      bulk_load(sld + 512, p.ws.D + row0, 4 * rows, full);
    }
    g += x.nch;
    ++tc;
  }
  return 0;
}

// S^T = K Q^T and dP^T = V dO^T for every chunk (warp 1, one thread).  S/dP of
// chunk G + 1 goes in as soon as the gradient warps hold chunk G's values in
// registers, so it overlaps their arithmetic and chunk G's gradient products.
template <int D>
__device__ int sdp_issuer(const Params& p, const Sched& sch, uint32_t base, uint32_t tmem) {
  using C = Cfg<D>;
  const uint32_t bar = base + C::oBar;
  constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false, false);  // K Q^T, V dO^T
  int g = 0, tc = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    if (x.nch == 0) continue;
    const int kvb = tc % C::NKV;
    const uint32_t sK = base + C::oK + kvb * 2 * C::kTile;
    const uint64_t dK = smem_desc_sw128(sK, 0, 1024), dV = smem_desc_sw128(sK + C::kTile, 0, 1024);
    if (!mbar_wait(bar + 8 * (C::bKVFull + kvb), (tc / C::NKV) & 1)) return kErrKVFull;
    for (int c = 0; c < x.nch; ++c) {
      const int G = g + c, st = G % C::NS;
      const uint32_t sQ = base + C::oQ + st * 2 * C::kTile;
      const uint64_t dQ = smem_desc_sw128(sQ, 0, 1024), ddO = smem_desc_sw128(sQ + C::kTile, 0, 1024);
      if (!mbar_wait(bar + 8 * (C::bQDFull + st), (G / C::NS) & 1)) return kErrQDFull;
      if (!mbar_wait(bar + 8 * C::bSDPFree, (G & 1) ^ 1)) return kErrSDPFree;
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = ((k >> 2) * kSlab + (k & 3) * 32) >> 4;  // descriptor address units
        mma_bf16_ss(tmem + C::tS, desc_add(dK, off), desc_add(dQ, off), kIdS, k > 0);
        mma_bf16_ss(tmem + C::tDP, desc_add(dV, off), desc_add(ddO, off), kIdS, k > 0);
      }
      mma_commit(bar + 8 * C::bSDPFull);
    }
    g += x.nch;
    ++tc;
  }
  return 0;
}

// dV += P^T dO, dK += dS^T Q and dQ_c = dS K for every chunk (warp 2, one
// thread).  The S/dP products of a chunk completed before its gradient warps
// began, so a commit here also covers every read of that chunk's Q/dO.
template <int D>
__device__ int grad_issuer(const Params& p, const Sched& sch, uint32_t base, uint32_t tmem) {
  using C = Cfg<D>;
  const uint32_t bar = base + C::oBar;
  constexpr uint32_t kIdKV = idesc_bf16_f32(128, D, false, true);  // P^T dO, dS^T Q
  constexpr uint32_t kIdQ = idesc_bf16_f32(128, D, true, true);    // dS K
  const uint64_t dSk = smem_desc_sw128(base + C::oDS, 0, 1024);      // dS^T, K-major A
  const uint64_t dSm = smem_desc_sw128(base + C::oDS, kSlab, 1024);  // dS, MN-major A
  int g = 0, tc = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    if (x.nch == 0) continue;
    const int kvb = tc % C::NKV;
    const uint64_t dK = smem_desc_sw128(base + C::oK + kvb * 2 * C::kTile, kSlab, 1024);
    for (int c = 0; c < x.nch; ++c) {
      const int G = g + c, st = G % C::NS;
      const uint32_t sQ = base + C::oQ + st * 2 * C::kTile;
      const uint64_t dQ = smem_desc_sw128(sQ, kSlab, 1024), ddO = smem_desc_sw128(sQ + C::kTile, kSlab, 1024);
      const bool acc = c > 0;
      if (!mbar_wait(bar + 8 * C::bPDSFull, G & 1)) return kErrPDSFull;
      if (c == 0 && !mbar_wait(bar + 8 * C::bDKVFree, (tc & 1) ^ 1)) return kErrDKVFree;
      if (!mbar_wait(bar + 8 * C::bDQFree, (G & 1) ^ 1)) return kErrDQFree;
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < kRows / 16; ++k) {  // k over the chunk's queries
        const uint32_t off = ((k >> 2) * kSlab + (k & 3) * 32) >> 4;
        const uint32_t mn = (k * 2048) >> 4;  // 16 rows of an MN-major operand
        mma_bf16_ts(tmem + C::tDV, tmem + C::tP + 8 * k, desc_add(ddO, mn), kIdKV, acc || k > 0);
        mma_bf16_ss(tmem + C::tDK, desc_add(dSk, off), desc_add(dQ, mn), kIdKV, acc || k > 0);
      }
      // Q and dO are last read by the products above: their buffer can refill
      // while the dQ product runs
      mma_commit(bar + 8 * (C::bQDFree + st));
#pragma unroll
      for (int k = 0; k < kRows / 16; ++k) {  // k over the tile's keys
        const uint32_t mn = (k * 2048) >> 4;
        mma_bf16_ss(tmem + C::tDQ, desc_add(dSm, mn), desc_add(dK, mn), kIdQ, k > 0);
      }
      mma_commit(bar + 8 * C::bPDSFree);
      mma_commit(bar + 8 * C::bDQFull);
      if (c == x.nch - 1) mma_commit(bar + 8 * C::bDKVFull);
    }
    g += x.nch;
    ++tc;
  }
  return 0;
}

// dK/dV tile stores (warp 3, one thread).  The gradient warps stage an item's
// dK and dV in the item's own K and V buffers (free once its last products
// have completed); the buffer is handed back to the producer once the stores
// have read it.
template <int D>
__device__ int out_storer(const Params& p, const Sched& sch, uint32_t base, const CUtensorMap* tdk,
                          const CUtensorMap* tdv) {
  using C = Cfg<D>;
  const uint32_t bar = base + C::oBar;
  int tc = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    if (x.nch == 0) continue;
    const int kvb = tc % C::NKV, bh = x.b * p.a.heads + x.h;
    const uint32_t sk = base + C::oK + kvb * 2 * C::kTile;
    if (!mbar_wait(bar + 8 * (C::bOutFull + kvb), (tc / C::NKV) & 1)) return kErrOutFull;
#pragma unroll
    for (int s = 0; s < D / 64; ++s) {
      tma_store_3d(tdk, sk + s * kSlab, s * 64, x.tile * kRows, bh);
      tma_store_3d(tdv, sk + C::kTile + s * kSlab, s * 64, x.tile * kRows, bh);
    }
    bulk_commit();
    bulk_wait_read0();
    mbar_arrive(bar + 8 * (C::bKVFree + kvb));
    ++tc;
  }
  bulk_wait_all0();  // the stores have landed before the CTA exits
  return 0;
}

// Gradient warps: thread = key row r; half hf owns query columns [64 hf, 64 hf + 64).
template <int D, bool kCausal>
__device__ int grad_warps(const Params& p, const Sched& sch, uint32_t base, uint8_t* gbase,
                          uint32_t tmem, int wq, int hf, int lane) {
  using C = Cfg<D>;
  const AttnArgs& a = p.a;
  const uint32_t bar = base + C::oBar;
  const int r = wq * 32 + lane;
  const uint32_t trow = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  const int nb = a.n / kBlock;
  const float sl2 = a.scale * kLog2e;
  auto all_ok = [](bool ok) { return __all_sync(0xffffffffu, ok); };
  // Epilogue: this thread's row of dK (first group, times 1/sqrt(d)) or dV
  // (second group) as packed bf16, then into the item's K (dK) or V (dV)
  // buffer as 128-byte swizzled boxes for the tile stores.
  uint32_t outp[D / 2];
  auto epi_load = [&](int etc, bool erow_valid) -> int {
    if (!all_ok(mbar_wait(bar + 8 * C::bDKVFull, etc & 1))) return kErrDKVFull;
    tc_fence_after();
    const float mul = erow_valid ? (hf == 0 ? a.scale : 1.f) : 0.f;
    const uint32_t tsrc = trow + (hf == 0 ? C::tDK : C::tDV);
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
    mbar_arrive(bar + 8 * C::bDKVFree);
    return 0;
  };
  auto epi_stage = [&](int ekvb) {
    uint8_t* stg = gbase + C::oK + ekvb * 2 * C::kTile + hf * C::kTile + r * 128;
#pragma unroll
    for (int gc = 0; gc < D / 8; ++gc)  // 16-byte chunk of the output row
      *reinterpret_cast<uint4*>(stg + (gc >> 3) * kSlab + (((gc & 7) ^ (r & 7)) << 4)) =
          make_uint4(outp[4 * gc], outp[4 * gc + 1], outp[4 * gc + 2], outp[4 * gc + 3]);
    fence_proxy_async_smem();
    mbar_arrive(bar + 8 * (C::bOutFull + ekvb));
  };
  struct Pend {
    bool valid;
    int tc;
    bool row_valid;
  } pend = {false, 0, false};
  int e = 0;
  // a key tile entirely past its sequence's length: dK = dV = 0 (first group dK, second dV)
  // (the tile's rows are contiguous: each group stores it as one coalesced run)
  auto zero_tile = [&](const Item& x) {
    const int64_t row0 = (static_cast<int64_t>(x.b) * a.heads + x.h) * a.n + x.tile * kRows;
    const int rows = min(kRows, a.n - x.tile * kRows);
    uint4* out = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(hf == 0 ? a.dk : a.dv) +
                                          row0 * D);
    for (int i = r; i < rows * (D / 8); i += 128) out[i] = make_uint4(0, 0, 0, 0);
  };
  int g = 0, tc = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    const int k = x.tile * kRows + r;
    if (x.nch == 0) {  // every key of the tile is padding
      zero_tile(x);
      continue;
    }
    const bool row_valid = k < x.L;
    const int kb = k / kBlock;
    for (int c = 0; c < x.nch; ++c) {
      const int G = g + c, st = G % C::NS;
      if (!all_ok(mbar_wait(bar + 8 * (C::bQDFull + st), (G / C::NS) & 1))) return kErrGQD;
      if (!all_ok(mbar_wait(bar + 8 * C::bSDPFull, G & 1))) return kErrSDPFull;
      tc_fence_after();
      const float* nl = reinterpret_cast<const float*>(gbase + C::oLD + st * 1024);
      const float* Dv = nl + 128;
      uint32_t wp[32], ws[32];  // packed bf16 P^T and dS^T for this thread's 64 queries
      float sa[2][32], dpa[2][32];
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        tmem_ld32(trow + C::tS + 64 * hf + 32 * jj, sa[jj]);
        tmem_ld32(trow + C::tDP + 64 * hf + 32 * jj, dpa[jj]);
      }
      tmem_wait_ld();
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        reg_fence(sa[jj]);
        reg_fence(dpa[jj]);
      }
      tc_fence_before();  // S and dP of this chunk are in registers: TMEM may be reused
      mbar_arrive(bar + 8 * C::bSDPFree);
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int j = 2 * hf + jj;  // 32-query group within the chunk
        const float(&s)[32] = sa[jj];
        const float(&dp)[32] = dpa[jj];
        const int qb = x.I0 + 4 * c + j;
        const bool vis = row_valid && qb < nb &&
                         (kCausal ? (qb >= kb && qb - kb <= a.R) : abs(qb - kb) <= a.R);
        // causal, diagonal block: queries before this key (index < k mod 32) see it not
        const int cut = kCausal && qb == kb ? (k & (kBlock - 1)) : 0;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          if (vis) {
            const float4 n0 = *reinterpret_cast<const float4*>(nl + 32 * j + 8 * cc);
            const float4 n1 = *reinterpret_cast<const float4*>(nl + 32 * j + 8 * cc + 4);
            const float4 d0 = *reinterpret_cast<const float4*>(Dv + 32 * j + 8 * cc);
            const float4 d1 = *reinterpret_cast<const float4*>(Dv + 32 * j + 8 * cc + 4);
            const float2 nv[4] = {make_float2(n0.x, n0.y), make_float2(n0.z, n0.w),
                                  make_float2(n1.x, n1.y), make_float2(n1.z, n1.w)};
            const float2 nd[4] = {make_float2(d0.x, d0.y), make_float2(d0.z, d0.w),
                                  make_float2(d1.x, d1.y), make_float2(d1.z, d1.w)};
            const float2 sl = make_float2(sl2, sl2);
#pragma unroll
            for (int e = 0; e < 4; ++e) {  // pairs of queries, packed fp32x2 arithmetic
              float2 x = __ffma2_rn(make_float2(s[8 * cc + 2 * e], s[8 * cc + 2 * e + 1]),
                                    sl, nv[e]);  // -inf for padding queries -> P = 0
              if (8 * cc + 2 * e < cut) x.x = -INFINITY;
              if (8 * cc + 2 * e + 1 < cut) x.y = -INFINITY;
              const float2 pe = make_float2(ex2_approx(x.x), ex2_approx(x.y));
              const float2 de = __fmul2_rn(
                  pe, __fadd2_rn(make_float2(dp[8 * cc + 2 * e], dp[8 * cc + 2 * e + 1]), nd[e]));
              wp[16 * jj + 4 * cc + e] = pack_bf16(pe.x, pe.y);
              ws[16 * jj + 4 * cc + e] = pack_bf16(de.x, de.y);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) wp[16 * jj + 4 * cc + e] = ws[16 * jj + 4 * cc + e] = 0u;
          }
        }
      }
      // the previous chunk's dV/dK/dQ products must be done reading the P/dS tiles
      if (!all_ok(mbar_wait(bar + 8 * C::bPDSFree, (G & 1) ^ 1))) return kErrPDSFree;

      uint8_t* srow = gbase + C::oDS + hf * kSlab + r * 128;
      // this thread's 64 queries = 32 packed columns of P^T in TMEM
      tmem_st32u(trow + C::tP + 32 * hf, wp);
#pragma unroll
      for (int jj = 0; jj < 2; ++jj)
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int ch = ((4 * jj + cc) ^ (r & 7)) << 4;
          *reinterpret_cast<uint4*>(srow + ch) =
              make_uint4(ws[16 * jj + 4 * cc], ws[16 * jj + 4 * cc + 1], ws[16 * jj + 4 * cc + 2],
                         ws[16 * jj + 4 * cc + 3]);
        }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar + 8 * C::bPDSFull);
      if (c == 0 && pend.valid) {
        // the previous item's epilogue: its last products completed before the
        // P/dS tiles were free, so only the TMEM read delays this chunk's products
        if ((e = epi_load(pend.tc, pend.row_valid))) return e;
        epi_stage(pend.tc % C::NKV);
        pend.valid = false;
      }
    }
    pend = {true, tc, row_valid};
    g += x.nch;
    ++tc;
  }
  if (pend.valid) {
    if ((e = epi_load(pend.tc, pend.row_valid))) return e;
    epi_stage(pend.tc % C::NKV);
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

// dQ warps: thread = query row of the chunk (warp w: rows 32 w .. 32 w + 31).
// Each warp stages its 32 rows of a 32-column box in its own 4 KB of the
// staging area and reduce-adds them with its own TMA bulk reduce, so the four
// warps never wait for one another.
template <int D>
__device__ int dq_warps(const Params& p, const Sched& sch, uint32_t base, uint8_t* gbase,
                        uint32_t tmem, int wq, int lane, const CUtensorMap* tdq) {
  using C = Cfg<D>;
  const AttnArgs& a = p.a;
  const uint32_t bar = base + C::oBar;
  const uint32_t trow = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  auto all_ok = [](bool ok) { return __all_sync(0xffffffffu, ok); };
  int g = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    if (x.nch == 0) continue;
    const int bh = x.b * a.heads + x.h;
    for (int c = 0; c < x.nch; ++c) {
      const int G = g + c;
      const int q0 = (x.I0 + 4 * c) * kBlock;
      if (!all_ok(mbar_wait(bar + 8 * C::bDQFull, G & 1))) return kErrDQFull;
      tc_fence_after();
      // dQ_c through the warp's staging box, one 32-column box per pass; the row is read
      // from TMEM 64 columns at a time and its TMEM released after the last read
      uint8_t* stg = gbase + C::oStg;
#pragma unroll
      for (int grp = 0; grp < D / 64; ++grp) {
        float v[2][32];
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) tmem_ld32(trow + C::tDQ + 64 * grp + 32 * jj, v[jj]);
        tmem_wait_ld();
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) reg_fence(v[jj]);
        if (grp == D / 64 - 1) {
          tc_fence_before();
          mbar_arrive(bar + 8 * C::bDQFree);
        }
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int j = 2 * grp + jj;  // 32-column box within the row
          // this warp's 32 rows go through its own 4 KB box and its own reduce-add
          if (lane == 0) bulk_wait_read0();  // the box's previous reduce-add has read it
          __syncwarp();
          uint8_t* box = stg + wq * 4096;
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<float4*>(box + lane * 128 + ((u ^ (lane & 7)) << 4)) =
                make_float4(v[jj][4 * u], v[jj][4 * u + 1], v[jj][4 * u + 2], v[jj][4 * u + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && q0 + 32 * wq < a.n) {
            tma_reduce_add_3d(tdq, base + C::oStg + wq * 4096, 32 * j, q0 + 32 * wq, bh);
            bulk_commit();
          }
        }
      }
    }
    g += x.nch;
  }
  if (lane == 0) bulk_wait_all0();  // the last reduce-adds have read shared memory and landed
  return 0;
}

template <int D, bool kCausal>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                       const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tdo,
                       const __grid_constant__ CUtensorMap tdq, const __grid_constant__ CUtensorMap tdk,
                       const __grid_constant__ CUtensorMap tdv, const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bar = base + C::oBar;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NKV; ++i) {
      mbar_init(bar + 8 * (C::bKVFull + i), 1);
      mbar_init(bar + 8 * (C::bKVFree + i), 1);
    }
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(bar + 8 * (C::bQDFull + i), 1);
      mbar_init(bar + 8 * (C::bQDFree + i), 1);
    }
    mbar_init(bar + 8 * C::bSDPFull, 1);
    mbar_init(bar + 8 * C::bSDPFree, 256);
    mbar_init(bar + 8 * C::bPDSFull, 256);
    mbar_init(bar + 8 * C::bPDSFree, 1);
    mbar_init(bar + 8 * C::bDQFull, 1);
    mbar_init(bar + 8 * C::bDQFree, 128);
    mbar_init(bar + 8 * C::bDKVFull, 1);
    mbar_init(bar + 8 * C::bDKVFree, 256);
    for (int i = 0; i < C::NKV; ++i) mbar_init(bar + 8 * (C::bOutFull + i), 256);
    mbar_init(bar + 8 * C::bDone, 2);  // one commit per MMA-issuing thread
    fence_barrier_init();
  }
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tk);
      prefetch_tmap(&tv);
      prefetch_tmap(&tq);
      prefetch_tmap(&tdo);
      prefetch_tmap(&tdq);
      prefetch_tmap(&tdk);
      prefetch_tmap(&tdv);
    }
  }
  if (warp == 1) {
    tmem_alloc(base + C::oSlot, C::kTmemCols);
    tmem_relinquish();
  }
  pdl_wait();  // everything above overlaps the previous kernel's tail
  if (warp == 0) sched_build(reinterpret_cast<int*>(gbase + C::oSched), p.a, kRows, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + C::oSlot);
  const Sched sch = sched_view(reinterpret_cast<const int*>(gbase + C::oSched), p.a, p.items);

  // Role branches never join again: each ends with the CTA barrier, after which
  // warp 1 waits for the tensor cores and frees the TMEM.
  if (warp < 4) {
    regs_dec<C::kRegsCtl, kLaunchRegs>();
    int err = 0;
    if (warp == 0 && lane == 0) err = producer<D>(p, sch, base, &tk, &tv, &tq, &tdo);
    if (warp == 1 && lane == 0) err = sdp_issuer<D>(p, sch, base, tmem);
    if (warp == 2 && lane == 0) err = grad_issuer<D>(p, sch, base, tmem);
    if (warp == 3 && lane == 0) err = out_storer<D>(p, sch, base, &tdk, &tdv);
    if (err) record_error(p.a.err, err);
    pdl_trigger();  // this CTA's work is issued: the next kernel may start launching
    __syncthreads();
    if (warp == 2 && lane == 0) mma_commit(bar + 8 * C::bDone);
    if (warp == 1) {
      if (lane == 0) {
        mma_commit(bar + 8 * C::bDone);
        if (!mbar_wait(bar + 8 * C::bDone, 0)) record_error(p.a.err, kErrDone);
      }
      __syncwarp();
      tc_fence_after();
      tmem_dealloc(tmem, C::kTmemCols);
    }
  } else if (warp < 12) {
    regs_inc<C::kRegsGrad, kLaunchRegs>();
    const int err =
        grad_warps<D, kCausal>(p, sch, base, gbase, tmem, warp & 3, (warp - 4) >> 2, lane);
    if (err) record_error(p.a.err, err);
    pdl_trigger();  // this CTA's work is issued: the next kernel may start launching
    __syncthreads();
  } else {
    regs_dec<C::kRegsDq, kLaunchRegs>();
    const int err = dq_warps<D>(p, sch, base, gbase, tmem, warp & 3, lane, &tdq);
    if (err) record_error(p.a.err, err);
    pdl_trigger();  // this CTA's work is issued: the next kernel may start launching
    __syncthreads();
  }
}

template <int D>
cudaError_t launch(const AttnArgs& a, int64_t rows, cudaStream_t stream) {
  using C = Cfg<D>;
  const int64_t heads_total = static_cast<int64_t>(a.batch) * a.heads;
  Params p;
  p.a = a;
  p.ws = bwd_workspace(a.workspace, rows);
  CUtensorMap tk, tv, tq, tdo, tdq, tdk, tdv;
  if (!make_tmap_bf16_rows(&tk, a.k, D, a.n, heads_total, kRows) ||
      !make_tmap_bf16_rows(&tv, a.v, D, a.n, heads_total, kRows) ||
      !make_tmap_bf16_rows(&tq, a.q, D, a.n, heads_total, kRows) ||
      !make_tmap_bf16_rows(&tdo, a.dout, D, a.n, heads_total, kRows) ||
      !make_tmap_rows(&tdq, p.ws.dqacc, true, D, a.n, heads_total, 32, 32) ||
      !make_tmap_bf16_rows(&tdk, a.dk, D, a.n, heads_total, kRows) ||
      !make_tmap_bf16_rows(&tdv, a.dv, D, a.n, heads_total, kRows))
    return cudaErrorInvalidValue;
  p.ntiles = (a.n + kRows - 1) / kRows;
  const int64_t items = heads_total * p.ntiles;
  if (items > (1ll << 30)) return cudaErrorInvalidValue;
  p.items = static_cast<int>(items);
  auto kernel = a.causal ? attn_bwd_tc_kernel<D, true> : attn_bwd_tc_kernel<D, false>;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(items < num_sms() ? items : num_sms());
  return launch_pdl(kernel, dim3(grid), dim3(kThreads), C::kSmem, stream, tk, tv, tq,
                    tdo, tdq, tdk, tdv, p);
}

}  // namespace

cudaError_t launch_bwd_main_tc(const AttnArgs& a, int64_t rows, cudaStream_t stream) {
  return a.d == 64 ? launch<64>(a, rows, stream) : launch_bwd_main_tc_d128(a, rows, stream);
}

}  // namespace nb
