// Banded block-sparse local attention forward for d = 64 on the
// 5th-generation tensor cores (tcgen05 + TMEM), bf16 in / fp32 accumulate,
// with two query tiles in flight per CTA.  (NucleoByte page, section 3: band
// |i - j| <= R over blocks of B = 32, scores Q K^T / sqrt(d), online softmax
// with running max, running sum and running output.)
//
// Work item = two consecutive 128-row query tiles, slots A and B (query
// blocks 8u .. 8u + 3 and 8u + 4 .. 8u + 7) of one (batch, head).  Their key
// windows overlap, so the item walks the union window in chunks of 128 keys
// (four key blocks) that both slots read from the same shared-memory stage:
// each K/V chunk is loaded once for up to two tiles.  Each slot has its own
// MMA-issuing thread, score buffer S (128 TMEM columns), output accumulator O
// (64 columns) and softmax warpgroup, so one slot's exponentials overlap the
// other slot's tensor-core work (S = Q K^T, then O += P V with P in TMEM).
//
// Softmax (thread = query row, all 128 keys of a chunk):
//   * the first chunk with a visible key takes the exact row max as the
//     reference m; later chunks compute P = 2^(s scale log2 e - m) against
//     the reference BEFORE knowing their own max, so the max no longer
//     precedes the exponentials.  A chunk whose sum exceeds 2^8 raises m by
//     the sum's binary exponent at the next chunk (O and l rescaled there,
//     after the previous P V has landed); a chunk whose sum exceeds 2^64
//     (scores far above the reference) is recomputed against its exact max.
//     Every P stays finite and the result is exact after the final O / l.
//   * a fixed share of the exponentials runs on the FMA pipe instead of the
//     special-function unit: 2^x = 2^n 2^f with n = round(x) by Cody and
//     Waite's range reduction and 2^f on [-1/2, 1/2] by a degree-3 polynomial
//     with constant term 1 whose other coefficients minimise the maximum
//     relative error (1.0e-4, far below the bf16 rounding of P), solved as a
//     linear program; x is clamped to [-127, 64] so that a masked key
//     (x = -inf) gives exactly 0.
//
// Warp roles (384 threads): warp 0 TMA producer (Q tiles, K/V chunks);
// warp 1 TMEM owner and issuer of slot A; warp 2 issuer of slot B; warps 4-7
// softmax and epilogue of slot A, warps 8-11 of slot B.  Epilogue: O / l in
// bf16 staged in swizzled shared memory and written by one TMA tensor store;
// lse = m + log2(l) in natural-log units.  Every wait is bounded; on a timeout
// the kernel records an error code in the caller-visible error word and tears
// down (frees TMEM) instead of hanging.
#include <math.h>

#include "nb_internal.h"
#include "schedule.cuh"
#include "sm100.cuh"

namespace nb {
namespace {

using namespace sm100;

constexpr int D = 64;
constexpr int kThreads = 384;
constexpr int kRows = 128;         // query rows per tile (slot)
constexpr int kItemRows = 256;     // query rows per work item (two slots)
constexpr int kChunk = 128;        // keys per chunk
constexpr int kSlab = 128 * 128;   // one swizzled box: 128 rows x 64 bf16
constexpr int NKV = 4;             // K/V chunk stages
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRaise = 256.f;                 // 2^8
constexpr float kRedo = 18446744073709551616.f;  // 2^64
// Exponentials of pairs e with (e & 7) < kEmu (of each block's 16 pairs) run
// on the FMA pipe: kEmu / 8 of them.
constexpr int kEmu = 2;

// smem layout (offsets from the 1024-byte aligned base)
constexpr int kQBytes = kRows * D * 2;   // 16 KB
constexpr int kKBytes = kChunk * D * 2;  // 16 KB
constexpr int oQ = 0;                    // slot s: oQ + s kQBytes
constexpr int oK = oQ + 2 * kQBytes;     // stage st: oK + st kKBytes
constexpr int oV = oK + NKV * kKBytes;
constexpr int oStg = oV + NKV * kKBytes;  // output staging, slot s: oStg + s kQBytes
constexpr int oBar = oStg + 2 * kQBytes;
constexpr int bQFull = 0, bQFree = 2, bKVFull = 4, bKVFree = bKVFull + NKV, bSFull = bKVFree + NKV,
              bPFull = bSFull + 2, bPVDone = bPFull + 2, bOFree = bPVDone + 2,
              bStgFree = bOFree + 2, bStgFull = bStgFree + 2, bDone = bStgFull + 2,
              nBar = bDone + 1;
constexpr int oSlot = oBar + nBar * 8;
constexpr int oSched = oSlot + 16;
constexpr int kSmem = oSched + kSchedBytes + 1024;
static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
constexpr uint32_t kTmemCols = 512;
__device__ __forceinline__ uint32_t tS(int s) { return s * 128; }       // S / P of slot s
__device__ __forceinline__ uint32_t tO(int s) { return 256 + s * 64; }  // O of slot s
// registers per thread after reallocation: control warpgroup, each softmax warpgroup
constexpr int kRegsCtl = 56, kRegsSoft = 224;
constexpr int kRegsLaunch = 168;  // 65536 / 384 rounded down to a multiple of 8
static_assert(128 * kRegsCtl + 256 * kRegsSoft <= kThreads * kRegsLaunch, "register budget");

struct Params {
  AttnArgs a;
  int nitems2;  // work items (256-row pairs of tiles) per (batch, head)
  int items;    // batch * heads * nitems2
};

struct Item {
  int b, h, u, L, J0, nch;
  int c0[2], c1[2];  // chunk range of each slot (c0 > c1: slot has no rows)
};

__device__ __forceinline__ Item decode_bht(const Params& p, int b, int h, int u) {
  const AttnArgs& a = p.a;
  Item x;
  x.b = b;
  x.h = h;
  x.u = u;
  int L = a.lengths ? a.lengths[b] : a.n;
  x.L = min(max(L, 0), a.n);
  const int nb = a.n / kBlock;
  x.J0 = 0;
  x.nch = 0;
  x.c0[0] = x.c0[1] = 1;
  x.c1[0] = x.c1[1] = 0;
  if (u * kItemRows >= x.L) return x;
  const int last = (x.L - 1) / kBlock;  // last block holding a valid query and key
  int hi_union = 0;
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    const int qb0 = 8 * u + 4 * s;
    if (qb0 > last) continue;
    const int lo = max(0, qb0 - a.R);
    const int hi = min(min(qb0 + 3, nb - 1) + (a.causal ? 0 : a.R), last);
    if (s == 0) x.J0 = lo;
    x.c0[s] = (lo - x.J0) / 4;
    x.c1[s] = (hi - x.J0) / 4;
    hi_union = hi;
  }
  x.nch = (hi_union - x.J0) / 4 + 1;
  return x;
}

__device__ __forceinline__ Item decode(const Params& p, int it) {
  const int bh = it / p.nitems2;
  const int b = bh / p.a.heads;
  return decode_bht(p, b, bh - b * p.a.heads, it - bh * p.nitems2);
}

__device__ __forceinline__ Item sched_item(const Params& p, const Sched& s, int k) {
  if (!s.balanced) return decode(p, k);
  int b, h, u;
  sched_nonempty(s, p.a.batch, p.a.heads, k, b, h, u);
  return decode_bht(p, b, h, u);
}

__device__ __forceinline__ bool slot_used(const Item& x, int s) { return x.c0[s] <= x.c1[s]; }

enum : int { kErrQFree = 0x41, kErrKVFree, kErrKVFull, kErrQFull, kErrPVPrev, kErrPFull, kErrOFree,
             kErrSFull, kErrPVLast, kErrStgFree, kErrStgFull, kErrDone };

__device__ int producer(const Params& p, const Sched& sch, uint32_t base, const CUtensorMap* tq,
                        const CUtensorMap* tk, const CUtensorMap* tv) {
  const uint32_t bar = base + oBar;
  int G = 0, qt[2] = {0, 0};
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    if (x.nch == 0) continue;
    const int bh = x.b * p.a.heads + x.h;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (!slot_used(x, s)) continue;
      if (!mbar_wait(bar + 8 * (bQFree + s), (qt[s] & 1) ^ 1)) return kErrQFree;
      mbar_arrive_expect_tx(bar + 8 * (bQFull + s), kQBytes);
      tma_load_3d(base + oQ + s * kQBytes, tq, bar + 8 * (bQFull + s), 0,
                  x.u * kItemRows + s * kRows, bh);
      ++qt[s];
    }
    for (int c = 0; c < x.nch; ++c, ++G) {
      const int st = G % NKV;
      if (!mbar_wait(bar + 8 * (bKVFree + st), ((G / NKV) & 1) ^ 1)) return kErrKVFree;
      const uint32_t full = bar + 8 * (bKVFull + st);
      mbar_arrive_expect_tx(full, 2 * kKBytes);
      const int y = (x.J0 + 4 * c) * kBlock;
      tma_load_3d(base + oK + st * kKBytes, tk, full, 0, y, bh);
      tma_load_3d(base + oV + st * kKBytes, tv, full, 0, y, bh);
    }
  }
  return 0;
}

// Issuer of slot s (one thread): per chunk of the item's union window, S = Q
// K^T then, once the softmax has written P, O (+)= P V.  A chunk the slot does
// not use is still waited for and released, so the stage's release count is
// two per chunk.  S of the next chunk waits for the previous P V (P lives in
// the S columns).
template <int s>
__device__ int issuer(const Params& p, const Sched& sch, uint32_t base, uint32_t tmem) {
  const uint32_t bar = base + oBar;
  constexpr uint32_t kIdS = idesc_bf16_f32(128, kChunk, false, false);  // Q K^T: both K-major
  constexpr uint32_t kIdPV = idesc_bf16_f32(128, D, false, true);       // V is MN-major
  const uint64_t dQ = smem_desc_sw128(base + oQ + s * kQBytes, 0, 1024);
  const uint32_t tSs = tmem + tS(s), tOs = tmem + tO(s);
  int G = 0, qt = 0, np = 0;  // union chunks seen, tiles of this slot, S/P rounds of this slot
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    if (x.nch == 0) continue;
    const bool used = slot_used(x, s);
    for (int c = 0; c < x.nch; ++c, ++G) {
      const int st = G % NKV;
      if (!mbar_wait(bar + 8 * (bKVFull + st), (G / NKV) & 1)) return kErrKVFull;
      if (used && c >= x.c0[s] && c <= x.c1[s]) {
        if (c == x.c0[s] && !mbar_wait(bar + 8 * (bQFull + s), qt & 1)) return kErrQFull;
        if (np > 0 && !mbar_wait(bar + 8 * (bPVDone + s), (np - 1) & 1)) return kErrPVPrev;
        tc_fence_after();
        const uint64_t dK = smem_desc_sw128(base + oK + st * kKBytes, 0, 1024);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_bf16_ss(tSs, desc_add(dQ, (k * 32) >> 4), desc_add(dK, (k * 32) >> 4), kIdS, k > 0);
        mma_commit(bar + 8 * (bSFull + s));
        if (c == x.c1[s]) mma_commit(bar + 8 * (bQFree + s));  // the tile's S products issued
        if (!mbar_wait(bar + 8 * (bPFull + s), np & 1)) return kErrPFull;
        if (c == x.c0[s] && qt > 0 && !mbar_wait(bar + 8 * (bOFree + s), (qt - 1) & 1))
          return kErrOFree;
        tc_fence_after();
        // V is MN-major: 8-key groups 1024 bytes apart, a 16-key step is 2048 bytes
        const uint64_t dV = smem_desc_sw128(base + oV + st * kKBytes, kSlab, 1024);
#pragma unroll
        for (int k = 0; k < kChunk / 16; ++k)
          mma_bf16_ts(tOs, tSs + 8 * k, desc_add(dV, (k * 2048) >> 4), kIdPV, c > x.c0[s] || k > 0);
        mma_commit(bar + 8 * (bPVDone + s));
        ++np;
      }
      mma_commit(bar + 8 * (bKVFree + st));
    }
    if (used) ++qt;
  }
  return 0;
}

// Softmax and epilogue warpgroup of slot s: thread = tile row r (TMEM lane r).
template <bool kCausal, int s>
__device__ int softmax(const Params& p, const Sched& sch, uint32_t base, uint8_t* gbase,
                       uint32_t tmem, int wq, int lane, const CUtensorMap* to) {
  const AttnArgs& a = p.a;
  const uint32_t bar = base + oBar;
  const int r = wq * 32 + lane;
  const uint32_t trow = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  const uint32_t tSr = trow + tS(s), tOr = trow + tO(s);
  const int nb = a.n / kBlock;
  const float sl2 = a.scale * kLog2e;
  const bool leader = r == 0;
  uint8_t* stg = gbase + oStg + s * kQBytes;
  auto all_ok = [](bool ok) { return __all_sync(0xffffffffu, ok); };
  // O and l times alpha (O is in TMEM; no P V product is in flight when called)
  auto rescale = [&](float alpha, float& l) {
#pragma unroll
    for (int j = 0; j < D / 32; ++j) {
      float ov[32];
      tmem_ld32(tOr + 32 * j, ov);
      tmem_wait_ld();
      reg_fence(ov);
#pragma unroll
      for (int i = 0; i < 32; ++i) ov[i] *= alpha;
      tmem_st32(tOr + 32 * j, ov);
    }
    tmem_wait_st();
    l *= alpha;
  };
  auto zero_rows = [&](int64_t row0, int rows, int nthreads, int t) {
    uint4* out = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(const_cast<void*>(a.o)) +
                                          row0 * D);
    for (int i = t; i < rows * (D / 8); i += nthreads) out[i] = make_uint4(0, 0, 0, 0);
    if (a.lse)
      for (int i = t; i < rows; i += nthreads) a.lse[row0 + i] = -INFINITY;
  };
  int np = 0, qt = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    const int64_t bh = static_cast<int64_t>(x.b) * a.heads + x.h;
    const int q0 = x.u * kItemRows + s * kRows;  // first row of this slot's tile
    if (!slot_used(x, s)) {  // this tile lies past the length: O = 0, lse = -inf
      if (q0 < a.n) zero_rows(bh * a.n + q0, min(kRows, a.n - q0), kRows, r);
      continue;
    }
    const int q = q0 + r;
    const int qb = q / kBlock;
    const bool row_valid = q < x.L;
    float m = -INFINITY, l = 0.f;  // reference max (base 2, scaled) and sum w.r.t. it
    int raise = 0;                 // pending increase of m (applied at the next chunk)
    for (int c = x.c0[s]; c <= x.c1[s]; ++c, ++np) {
      if (!all_ok(mbar_wait(bar + 8 * (bSFull + s), np & 1))) return kErrSFull;
      tc_fence_after();
      float sc[4][32];
#pragma unroll
      for (int j = 0; j < 4; ++j) tmem_ld32(tSr + 32 * j, sc[j]);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 4; ++j) reg_fence(sc[j]);
      // the previous chunk's P V has landed (S of this chunk was issued after it)
      if (__any_sync(0xffffffffu, raise != 0)) {
        const float alpha = raise != 0 ? ex2_approx(-static_cast<float>(raise)) : 1.f;
        m += static_cast<float>(raise);
        rescale(alpha, l);
        raise = 0;
      }
      bool vis[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int kb = x.J0 + 4 * c + j;
        vis[j] = row_valid && kb < nb && kb * kBlock < x.L &&
                 (kCausal ? (kb <= qb && qb - kb <= a.R) : abs(kb - qb) <= a.R);
        if (vis[j]) {
          // keys at or past the length are masked, and (causal) keys after the query
          const int lim = min(x.L - kb * kBlock, kCausal && kb == qb ? q - kb * kBlock + 1 : kBlock);
          if (lim < 32) {
#pragma unroll
            for (int i = 0; i < 32; ++i) sc[j][i] = i < lim ? sc[j][i] : -INFINITY;
          }
        }
      }
      auto row_max = [&]() {
        float pm[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) pm[i] = -INFINITY;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (vis[j])
#pragma unroll
            for (int i = 0; i < 32; ++i) pm[i & 7] = fmaxf(pm[i & 7], sc[j][i]);
        return fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                     fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7]))) * sl2;
      };
      if (m == -INFINITY) m = row_max();  // first chunk with a visible key: exact max
      // P = 2^(s sl2 - m) in bf16 over the S columns; sum into lsum
      float lsum = 0.f;
      auto exps = [&](bool store) {
        const float2 nm = make_float2(-m, -m);
        const float2 sl = make_float2(sl2, sl2);
        float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        const bool live = m != -INFINITY;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t w[16];
          if (vis[j] && live) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float2 xv = __ffma2_rn(make_float2(sc[j][2 * e], sc[j][2 * e + 1]), sl, nm);
              const float2 pv = (e & 7) < kEmu ? exp2_fma(xv)
                                               : make_float2(ex2_approx(xv.x), ex2_approx(xv.y));
              acc[e & 1] = __fadd2_rn(acc[e & 1], pv);
              w[e] = pack_bf16(pv.x, pv.y);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = 0u;
          }
          if (store) tmem_st16u(tSr + 16 * j, w);
        }
        lsum = (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y);
      };
      exps(true);
      // a sum far above the reference (or not finite): this chunk again against
      // its exact max (warp-uniform: the TMEM accesses are warp-wide)
      if (__any_sync(0xffffffffu, !(lsum <= kRedo))) {
        const float cm = row_max();
        const bool up = cm > m;
        rescale(up ? ex2_approx(m - cm) : 1.f, l);
        if (up) m = cm;
        exps(true);
      }
      l += lsum;
      if (lsum > kRaise) raise = (__float_as_int(lsum) >> 23) - 127;  // floor(log2(lsum))
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar + 8 * (bPFull + s));
    }
    // epilogue: the tile's last P V product, then O / l
    if (!all_ok(mbar_wait(bar + 8 * (bPVDone + s), (np - 1) & 1))) return kErrPVLast;
    tc_fence_after();
    float o[2][32];
#pragma unroll
    for (int j = 0; j < 2; ++j) tmem_ld32(tOr + 32 * j, o[j]);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 2; ++j) reg_fence(o[j]);
    tc_fence_before();
    mbar_arrive(bar + 8 * (bOFree + s));
    const bool has = l > 0.f;  // padding rows and rows without a visible key: 0
    const float inv = has ? 1.f / l : 0.f;
    if (leader) {  // the previous tile's store has read the staging
      bulk_wait_read0();
      mbar_arrive(bar + 8 * (bStgFree + s));
    }
    if (!all_ok(mbar_wait(bar + 8 * (bStgFree + s), qt & 1))) return kErrStgFree;
#pragma unroll
    for (int gc = 0; gc < D / 8; ++gc) {  // 16-byte chunk gc of the row, swizzled
      const float* v = &o[gc >> 2][8 * (gc & 3)];
      *reinterpret_cast<uint4*>(stg + r * 128 + ((gc ^ (r & 7)) << 4)) =
          make_uint4(pack_bf16(v[0] * inv, v[1] * inv), pack_bf16(v[2] * inv, v[3] * inv),
                     pack_bf16(v[4] * inv, v[5] * inv), pack_bf16(v[6] * inv, v[7] * inv));
    }
    if (q < a.n && a.lse) a.lse[bh * a.n + q] = has ? (m + log2f(l)) * kLn2 : -INFINITY;
    fence_proxy_async_smem();
    mbar_arrive(bar + 8 * (bStgFull + s));
    if (leader) {
      if (!mbar_wait(bar + 8 * (bStgFull + s), qt & 1)) return kErrStgFull;
      tma_store_3d(to, base + oStg + s * kQBytes, 0, q0, static_cast<int>(bh));
      bulk_commit();
    }
    ++qt;
  }
  if (leader) bulk_wait_all0();  // the last tile's store has landed before the CTA exits
  if (sch.balanced) {            // second pass: items past their sequence's length
    for (int e = blockIdx.x; e < p.items - sch.count; e += gridDim.x) {
      int b, h, u;
      sched_empty(sch, a.batch, a.heads, p.nitems2, e, b, h, u);
      const int64_t row0 = (static_cast<int64_t>(b) * a.heads + h) * a.n + u * kItemRows;
      const int rows = min(kItemRows, a.n - u * kItemRows);
      zero_rows(row0, rows, 2 * kRows, s * kRows + r);
    }
  }
  return 0;
}

template <bool kCausal>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_pp_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to,
                       const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bar = base + oBar;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar + 8 * (bQFull + i), 1);
      mbar_init(bar + 8 * (bQFree + i), 1);
      mbar_init(bar + 8 * (bSFull + i), 1);
      mbar_init(bar + 8 * (bPFull + i), 128);
      mbar_init(bar + 8 * (bPVDone + i), 1);
      mbar_init(bar + 8 * (bOFree + i), 128);
      mbar_init(bar + 8 * (bStgFree + i), 1);
      mbar_init(bar + 8 * (bStgFull + i), 128);
    }
    for (int i = 0; i < NKV; ++i) {
      mbar_init(bar + 8 * (bKVFull + i), 1);
      mbar_init(bar + 8 * (bKVFree + i), 2);  // one release per issuer
    }
    mbar_init(bar + 8 * bDone, 2);  // one commit per issuer
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tq);
    prefetch_tmap(&tk);
    prefetch_tmap(&tv);
    prefetch_tmap(&to);
  }
  if (warp == 1) {
    tmem_alloc(base + oSlot, kTmemCols);
    tmem_relinquish();
  }
  pdl_wait();  // everything above overlaps the previous kernel's tail
  if (warp == 0) sched_build(reinterpret_cast<int*>(gbase + oSched), p.a, kItemRows, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + oSlot);
  const Sched sch = sched_view(reinterpret_cast<const int*>(gbase + oSched), p.a, p.items);

  // Role branches end with the CTA barrier, after which warp 1 waits for the
  // tensor cores and frees the TMEM.
  int err = 0;
  if (warp < 4) {
    regs_dec<kRegsCtl>();
    if (warp == 0 && lane == 0) err = producer(p, sch, base, &tq, &tk, &tv);
    if (warp == 1 && lane == 0) err = issuer<0>(p, sch, base, tmem);
    if (warp == 2 && lane == 0) err = issuer<1>(p, sch, base, tmem);
  } else {
    regs_inc<kRegsSoft>();
    err = warp < 8 ? softmax<kCausal, 0>(p, sch, base, gbase, tmem, warp & 3, lane, &to)
                   : softmax<kCausal, 1>(p, sch, base, gbase, tmem, warp & 3, lane, &to);
  }
  if (err) record_error(p.a.err, err);
  pdl_trigger();  // this CTA's work is issued: the next kernel may start launching
  __syncthreads();
  if (warp == 2 && lane == 0) mma_commit(bar + 8 * bDone);
  if (warp == 1) {
    if (lane == 0) {  // every tensor-core operation of this CTA has completed
      mma_commit(bar + 8 * bDone);
      if (!mbar_wait(bar + 8 * bDone, 0)) record_error(p.a.err, kErrDone);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_attn_fwd_pp(const AttnArgs& a, cudaStream_t stream) {
  if (a.d != D) return cudaErrorInvalidValue;
  const int64_t heads_total = static_cast<int64_t>(a.batch) * a.heads;
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_bf16_rows(&tq, a.q, D, a.n, heads_total, kRows) ||
      !make_tmap_bf16_rows(&tk, a.k, D, a.n, heads_total, kChunk) ||
      !make_tmap_bf16_rows(&tv, a.v, D, a.n, heads_total, kChunk) ||
      !make_tmap_bf16_rows(&to, a.o, D, a.n, heads_total, kRows))
    return cudaErrorInvalidValue;
  Params p;
  p.a = a;
  p.nitems2 = (a.n + kItemRows - 1) / kItemRows;
  const int64_t items = heads_total * p.nitems2;
  if (items > (1ll << 30)) return cudaErrorInvalidValue;
  p.items = static_cast<int>(items);
  auto kernel = a.causal ? attn_fwd_pp_kernel<true> : attn_fwd_pp_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(items < num_sms() ? items : num_sms());
  return launch_pdl(kernel, dim3(grid), dim3(kThreads), kSmem, stream, tq, tk, tv, to, p);
}

}  // namespace nb
