// Banded block-sparse local attention forward on the 5th-generation tensor
// cores (tcgen05 + TMEM), bf16 in / fp32 accumulate.  (NucleoByte page,
// section 3: band |i - j| <= R over blocks of B = 32, scores Q K^T / sqrt(d),
// online softmax with running max, running sum and running output.)
//
// Work item = one query tile of 128 rows (four query blocks) of one (batch,
// head).  The union of the four bands is the key-block window
// [4t - R, 4t + 3 + R] ([4t - R, 4t + 3] for the causal band, the kCausal
// instantiation, which also masks keys after their query in the diagonal
// block) (clipped to the sequence and its length), processed in
// chunks of 128 keys (four key blocks).  A persistent grid of one CTA per SM
// walks the items; consecutive CTAs take neighbouring tiles at the same time,
// so the key/value blocks their windows share are served from L2.
//
// Warp roles (512 threads, four warpgroups with reallocated registers):
//   warp 0     TMA producer: Q tile, then K chunks, into 128-byte swizzled
//              shared memory (3-D tensor maps; rows outside [0, n) are
//              zero-filled by TMA and masked).  A K stage is freed as soon as
//              its S product completes.
//   warp 3     TMA producer of the V chunks (a V stage is freed by the P V
//              products, later than the K stage of the same chunk).
//   warp 1     TMEM owner and S issuer (one thread):
//                S_c = Q K_c^T   (M 128, N 128, K d)   -> TMEM, three buffers at
//                d = 64 (S of chunks c + 1 and c + 2 in flight while chunk c's
//                softmax runs), two at d = 128
//   warp 2     P V issuer (one thread):
//                O_h += P_c,h V_c,h  (M 128, N d, K 64; P read from TMEM)
//              Two issuing threads keep the tensor pipe fed: a lone thread
//              issuing both streams serialises every wait and commit with
//              the MMAs.
//   warps 4-11 softmax, two groups of four warps; thread (r, half) owns row r
//              (TMEM lane r) and 64 of the chunk's 128 key columns.  Per chunk
//              it reads its 64 scores, masks keys outside its query block's
//              band or past the length, updates its own running max and sum
//              (base 2) and writes P = 2^(s - m) as bf16 back into TMEM over
//              the scores it has read.  Each half keeps its own running output
//              O_h in TMEM; it is rescaled (load, multiply, store) only when
//              that half's max grows by more than 2^8, otherwise the stale max
//              is kept (P <= 2^8, exact after the final division).  At the end
//              of a tile each half hands its (m, l) of the row to the epilogue
//              warps through shared memory and goes on to the next tile.
//   warps 12-15 epilogue, thread = row: combine the halves
//              O = (O_0 2^(m_0 - M) + O_1 2^(m_1 - M)) / l, lse = M + log l;
//              the bf16 tile is staged in swizzled shared memory and written
//              by one TMA tensor store (coalesced, asynchronous).  The next
//              tile's first P V product waits until these warps have read O;
//              the softmax of that tile's first chunks does not.
// Every mbarrier wait is bounded; on a timeout the kernel records an error
// code in the caller-visible error word and tears down (frees TMEM) instead
// of hanging.
#include <math.h>

#include "nb_internal.h"
#include "schedule.cuh"
#include "sm100.cuh"

namespace nb {
namespace {

using namespace sm100;

constexpr int kThreads = 512;
constexpr int kLaunchRegs = 65536 / kThreads / 8 * 8;  // per thread at launch
constexpr int kRows = 128;   // query rows per tile
constexpr int kChunk = 128;  // keys per chunk
constexpr int kSlab = 128 * 128;  // one swizzled box: 128 rows x 64 bf16
constexpr float kTau = 8.0f;      // lazy-rescale threshold, log2 units
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D>
struct Cfg {
  static constexpr int NQ = D == 64 ? 2 : 1;   // Q tile buffers
  static constexpr int NKV = D == 64 ? 3 : 2;  // K chunk stages, and as many V chunk stages
  static constexpr int NSB = D == 64 ? 3 : 2;  // S buffers
  static constexpr int NOB = 1;  // O accumulators per half (tiles in flight)
  static constexpr int kQBytes = kRows * D * 2;
  static constexpr int kKBytes = kChunk * D * 2;
  static constexpr int oQ = 0;
  static constexpr int oK = oQ + NQ * kQBytes;
  static constexpr int oV = oK + NKV * kKBytes;
  static constexpr int oStg = oV + NKV * kKBytes;  // output tile staging (D / 64 boxes)
  static constexpr int oBar = oStg + kRows * D * 2;
  // barrier indices ([S buffer][half] for P, [half][buffer] for O)
  static constexpr int bQFull = 0, bQFree = bQFull + NQ, bKFull = bQFree + NQ,
                       bKFree = bKFull + NKV, bVFull = bKFree + NKV, bVFree = bVFull + NKV,
                       bSFull = bVFree + NKV, bSFree = bSFull + NSB,
                       bPFull = bSFree + NSB, bPVDone = bPFull + 2 * NSB, bOFull = bPVDone + 2 * NSB,
                       bOFree = bOFull + 2 * NOB, bXFull = bOFree + 2 * NOB, bXFree = bXFull + 2,
                       bDone = bXFree + 2, nBar = bDone + 1;
  static constexpr int oSlot = oBar + nBar * 8;
  // per-tile hand-off of the halves' running max and sum to the epilogue warps:
  // [parity][half][m, l][row] fp32
  static constexpr int oXSum = oSlot + 16;
  static constexpr int oSched = oXSum + 2 * 2 * 2 * 128 * 4;  // work-order prefix table
  static constexpr int kSmem = oSched + kSchedBytes + 1024;  // + slack for 1024-byte alignment
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
  static constexpr uint32_t kTmemCols = 512;
  // S buffer i: columns [128 i, 128 i + 128).  Half h's P (64 keys, two bf16
  // per column) overwrites the first 32 columns of that half's 64 S columns.
  // The O accumulators follow (d = 64: 384 + 2 x 64 columns; d = 128: 256 +
  // 2 x 128).
  static constexpr uint32_t tS = 0;
  __device__ static constexpr uint32_t tP(int sb, int h) { return tS + sb * kChunk + 64 * h; }
  // O accumulator of half h, buffer ob
  __device__ static constexpr uint32_t tO(int h, int ob) { return NSB * kChunk + (h * NOB + ob) * D; }
  static_assert(NSB * kChunk + 2 * NOB * D <= kTmemCols, "tensor memory columns");
  // registers per thread after reallocation: TMA/MMA warpgroup, each softmax
  // warpgroup, epilogue warpgroup (the 16 warps share the 64K-register file;
  // the d = 128 softmax spills less with 176, the d = 64 one runs faster at 168)
  static constexpr int kRegsCtl = 56;
  static constexpr int kRegsSoft = D == 64 ? 168 : 176;
  static constexpr int kRegsEpi = D == 64 ? 120 : 104;
  static_assert(128 * (kRegsCtl + 2 * kRegsSoft + kRegsEpi) <= 65536, "register budget");
};

struct Params {
  AttnArgs a;
  int ntiles;  // query tiles per (batch, head)
  int items;   // batch * heads * ntiles
};

struct Item {
  int b, h, tile, L, J0, nch;
};

__device__ __forceinline__ Item decode_bht(const Params& p, int b, int h, int tile, int L) {
  const AttnArgs& a = p.a;
  Item x;
  x.b = b;
  x.h = h;
  x.tile = tile;
  x.L = L;  // clamped to [0, n]
  const int nb = a.n / kBlock;
  x.J0 = 0;
  x.nch = 0;
  if (x.tile * kRows < x.L) {
    const int qb_last = min(x.tile * 4 + 3, nb - 1);
    x.J0 = max(0, x.tile * 4 - a.R);
    const int J1 = min(min(qb_last + (a.causal ? 0 : a.R), nb - 1), (x.L - 1) / kBlock);
    x.nch = (J1 - x.J0 + 4) / 4;
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

// error codes: 0x10 + site
enum : int { kErrQFree = 0x11, kErrKFree, kErrQFull, kErrKFull, kErrSFree, kErrOFree, kErrPFull,
             kErrSFull, kErrPPrev = 0x1a, kErrOFull, kErrDone, kErrXFull = 0x1e, kErrXFree, kErrVFree, kErrVFull };

template <int D>
__device__ int producer(const Params& p, const Sched& sch, uint32_t base, const CUtensorMap* tq,
                        const CUtensorMap* tk, const CUtensorMap* tv) {
  using C = Cfg<D>;
  const uint32_t bar = base + C::oBar;
  int g = 0, tc = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    if (x.nch == 0) continue;
    const int bh = x.b * p.a.heads + x.h;
    const int qs = tc % C::NQ;
    if (!mbar_wait(bar + 8 * (C::bQFree + qs), ((tc / C::NQ) & 1) ^ 1)) return kErrQFree;
    mbar_arrive_expect_tx(bar + 8 * (C::bQFull + qs), C::kQBytes);
#pragma unroll
    for (int s = 0; s < D / 64; ++s)
      tma_load_3d(base + C::oQ + qs * C::kQBytes + s * kSlab, tq, bar + 8 * (C::bQFull + qs),
                  s * 64, x.tile * kRows, bh);
    for (int c = 0; c < x.nch; ++c) {
      const int G = g + c, st = G % C::NKV;
      if (!mbar_wait(bar + 8 * (C::bKFree + st), ((G / C::NKV) & 1) ^ 1)) return kErrKFree;
      const uint32_t full = bar + 8 * (C::bKFull + st);
      mbar_arrive_expect_tx(full, C::kKBytes);
      const int y = (x.J0 + 4 * c) * kBlock;
#pragma unroll
      for (int s = 0; s < D / 64; ++s)
        tma_load_3d(base + C::oK + st * C::kKBytes + s * kSlab, tk, full, s * 64, y, bh);
    }
    g += x.nch;
    ++tc;
  }
  return 0;
}

// V chunks (warp 3, one thread).  A V stage is freed by the chunk's P V
// products, a K stage already by its S product, so the two streams run on
// their own: the next K chunks load while earlier P V products still read V.
template <int D>
__device__ int v_producer(const Params& p, const Sched& sch, uint32_t base, const CUtensorMap* tv) {
  using C = Cfg<D>;
  const uint32_t bar = base + C::oBar;
  int g = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    if (x.nch == 0) continue;
    const int bh = x.b * p.a.heads + x.h;
    for (int c = 0; c < x.nch; ++c) {
      const int G = g + c, st = G % C::NKV;
      if (!mbar_wait(bar + 8 * (C::bVFree + st), ((G / C::NKV) & 1) ^ 1)) return kErrVFree;
      const uint32_t full = bar + 8 * (C::bVFull + st);
      mbar_arrive_expect_tx(full, C::kKBytes);
      const int y = (x.J0 + 4 * c) * kBlock;
#pragma unroll
      for (int s = 0; s < D / 64; ++s)
        tma_load_3d(base + C::oV + st * C::kKBytes + s * kSlab, tv, full, s * 64, y, bh);
    }
    g += x.nch;
  }
  return 0;
}

// S = Q K^T for every chunk into S buffer G % NSB (warp 1, one thread).  P of
// chunk G replaces S in that buffer, so S of chunk G + NSB waits for P V of
// chunk G, which the other issuer signals on bSFree.
template <int D>
__device__ int s_issuer(const Params& p, const Sched& sch, uint32_t base, uint32_t tmem) {
  using C = Cfg<D>;
  const uint32_t bar = base + C::oBar;
  constexpr uint32_t kIdS = idesc_bf16_f32(128, kChunk, false, false);  // Q K^T: both K-major
  int g = 0, tc = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    if (x.nch == 0) continue;
    const int qs = tc % C::NQ;
    if (!mbar_wait(bar + 8 * (C::bQFull + qs), (tc / C::NQ) & 1)) return kErrQFull;
    const uint64_t dQ = smem_desc_sw128(base + C::oQ + qs * C::kQBytes, 0, 1024);
    for (int c = 0; c < x.nch; ++c) {
      const int G = g + c, st = G % C::NKV, sb = G % C::NSB;
      const uint64_t dK = smem_desc_sw128(base + C::oK + st * C::kKBytes, 0, 1024);
      const uint32_t tD = tmem + C::tS + sb * kChunk;
      if (!mbar_wait(bar + 8 * (C::bKFull + st), (G / C::NKV) & 1)) return kErrKFull;
      if (!mbar_wait(bar + 8 * (C::bSFree + sb), ((G / C::NSB) & 1) ^ 1)) return kErrSFree;
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = ((k >> 2) * kSlab + (k & 3) * 32) >> 4;  // descriptor address units
        mma_bf16_ss(tD, desc_add(dQ, off), desc_add(dK, off), kIdS, k > 0);
      }
      mma_commit(bar + 8 * (C::bSFull + sb));
      mma_commit(bar + 8 * (C::bKFree + st));  // the S product was this K chunk's only reader
      if (c == x.nch - 1) mma_commit(bar + 8 * (C::bQFree + qs));  // the tile's S products issued
    }
    g += x.nch;
    ++tc;
  }
  return 0;
}

// O_h += P_h V_h for every chunk and half (warp 10, one thread): P from TMEM,
// V from shared memory.  Completion of chunk G's products frees its S buffer
// and its K/V stage (S of chunk G completed before its softmax began).
template <int D>
__device__ int pv_issuer(const Params& p, const Sched& sch, uint32_t base, uint32_t tmem) {
  using C = Cfg<D>;
  const uint32_t bar = base + C::oBar;
  constexpr uint32_t kIdPV = idesc_bf16_f32(128, D, false, true);  // V is MN-major (K = 64 per half)
  int g = 0, tc = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    if (x.nch == 0) continue;
    const int ob = tc % C::NOB;
    for (int c = 0; c < x.nch; ++c) {
      const int G = g + c, st = G % C::NKV, sb = G % C::NSB;
      // V is MN-major: 64-column swizzle atoms kSlab apart, 8-key groups 1024 bytes apart
      const uint64_t dV = smem_desc_sw128(base + C::oV + st * C::kKBytes, kSlab, 1024);
      if (!mbar_wait(bar + 8 * (C::bVFull + st), (G / C::NKV) & 1)) return kErrVFull;
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // each half's 64 keys into its own O accumulator
        const uint32_t tO = tmem + C::tO(h, ob), tP = tmem + C::tP(sb, h);
        if (c == 0 &&
            !mbar_wait(bar + 8 * (C::bOFree + h * C::NOB + ob), ((tc / C::NOB) & 1) ^ 1))
          return kErrOFree;
        if (!mbar_wait(bar + 8 * (C::bPFull + 2 * sb + h), (G / C::NSB) & 1)) return kErrPFull;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 4; ++k)  // 16 keys = 8 P columns = 2048 bytes of V per step
          mma_bf16_ts(tO, tP + 8 * k, desc_add(dV, (h * 8192 + k * 2048) >> 4), kIdPV, c > 0 || k > 0);
        mma_commit(bar + 8 * (C::bPVDone + 2 * sb + h));
        if (c == x.nch - 1) mma_commit(bar + 8 * (C::bOFull + h * C::NOB + ob));
      }
      mma_commit(bar + 8 * (C::bSFree + sb));
      mma_commit(bar + 8 * (C::bVFree + st));
    }
    g += x.nch;
    ++tc;
  }
  return 0;
}

template <int D, bool kCausal>
__device__ int softmax_warps(const Params& p, const Sched& sch, uint32_t base, uint8_t* gbase,
                             uint32_t tmem, int wq, int hf, int lane) {
  using C = Cfg<D>;
  const AttnArgs& a = p.a;
  const uint32_t bar = base + C::oBar;
  const int r = wq * 32 + lane;  // tile row == TMEM lane
  const uint32_t trow = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  const int nb = a.n / kBlock;
  const float sl2 = a.scale * kLog2e;
  float* xs = reinterpret_cast<float*>(gbase + C::oXSum);
  auto all_ok = [](bool ok) { return __all_sync(0xffffffffu, ok); };
  // a tile entirely past its sequence's length: O = 0, lse = -inf
  // (the tile's rows are contiguous: the 256 threads store it as one coalesced run)
  auto zero_tile = [&](const Item& x) {
    const int64_t row0 = (static_cast<int64_t>(x.b) * a.heads + x.h) * a.n + x.tile * kRows;
    const int rows = min(kRows, a.n - x.tile * kRows);
    uint4* out = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(const_cast<void*>(a.o)) +
                                          row0 * D);
    for (int i = hf * 128 + r; i < rows * (D / 8); i += 256) out[i] = make_uint4(0, 0, 0, 0);
    if (a.lse && hf == 0 && r < rows) a.lse[row0 + r] = -INFINITY;
  };
  int g = 0, tc = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    const int q = x.tile * kRows + r;
    if (x.nch == 0) {  // the whole tile is padding
      zero_tile(x);
      continue;
    }
    const int qb = q / kBlock;
    const bool row_valid = q < x.L;
    const int ob = tc % C::NOB;
    float m_used = -INFINITY, l = 0.f;
    for (int c = 0; c < x.nch; ++c) {
      const int G = g + c, sb = G % C::NSB;
      if (!all_ok(mbar_wait(bar + 8 * (C::bSFull + sb), (G / C::NSB) & 1))) return kErrSFull;
      tc_fence_after();
      float s[2][32];
#pragma unroll
      for (int j = 0; j < 2; ++j) tmem_ld32(trow + C::tS + sb * kChunk + 64 * hf + 32 * j, s[j]);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 2; ++j) reg_fence(s[j]);

      bool vis[2];
      float pm[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) pm[i] = -INFINITY;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int kb = x.J0 + 4 * c + 2 * hf + j;
        vis[j] = row_valid && kb < nb && kb * kBlock < x.L &&
                 (kCausal ? (kb <= qb && qb - kb <= a.R) : abs(kb - qb) <= a.R);
        if (vis[j]) {
          // keys at or past the length are masked, and (causal) keys after the query
          const int lim = min(x.L - kb * kBlock, kCausal && kb == qb ? q - kb * kBlock + 1 : kBlock);
          if (lim < 32) {
#pragma unroll
            for (int i = 0; i < 32; ++i) s[j][i] = i < lim ? s[j][i] : -INFINITY;
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) pm[i & 7] = fmaxf(pm[i & 7], s[j][i]);
        }
      }
      // this half's running max (raw scores times the positive scale, base 2)
      const float cmax = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                               fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7]))) * sl2;
      bool need = false;
      float alpha = 1.f;
      if (cmax > m_used + kTau) {
        if (m_used != -INFINITY) {
          need = true;
          alpha = ex2_approx(m_used - cmax);
        }
        m_used = cmax;
      }
      // P = 2^(s scale log2e - m) in bf16 for this half's 64 keys
      const float2 nm = make_float2(-m_used, -m_used);
      const float2 sl = make_float2(sl2, sl2);
      uint32_t w[32];  // P of keys 2i, 2i + 1 of this half in w[i]
      float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        if (vis[j]) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {  // pairs of keys, packed fp32x2 arithmetic
            const float2 xv = __ffma2_rn(make_float2(s[j][2 * i], s[j][2 * i + 1]), sl, nm);
            const float2 pv = make_float2(ex2_approx(xv.x), ex2_approx(xv.y));
            ls[i & 1] = __fadd2_rn(ls[i & 1], pv);
            w[16 * j + i] = pack_bf16(pv.x, pv.y);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) w[16 * j + i] = 0u;
        }
      }
      if (__any_sync(0xffffffffu, need)) {
        // this half's previous P V product must have landed before its O is rescaled
        // (need implies c > 0, so chunk G - 1 belongs to this tile)
        const int Gp = G - 1;
        if (!all_ok(mbar_wait(bar + 8 * (C::bPVDone + 2 * (Gp % C::NSB) + hf), (Gp / C::NSB) & 1)))
          return kErrPPrev;
        tc_fence_after();
        const uint32_t to = trow + C::tO(hf, ob);
#pragma unroll
        for (int j = 0; j < D / 32; ++j) {
          float ov[32];
          tmem_ld32(to + 32 * j, ov);
          tmem_wait_ld();
          reg_fence(ov);
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] *= alpha;
          tmem_st32(to + 32 * j, ov);
        }
        tmem_wait_st();
        l *= alpha;
      }
      l += (ls[0].x + ls[0].y) + (ls[1].x + ls[1].y);
      // P over this half's S columns (already read into registers)
      tmem_st32u(trow + C::tP(sb, hf), w);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar + 8 * (C::bPFull + 2 * sb + hf));
    }
    // hand this half's (m, l) of the row to the epilogue warps
    const int par = tc & 1;
    if (!all_ok(mbar_wait(bar + 8 * (C::bXFree + par), ((tc >> 1) & 1) ^ 1))) return kErrXFree;
    xs[((par * 2 + hf) * 2 + 0) * 128 + r] = m_used;
    xs[((par * 2 + hf) * 2 + 1) * 128 + r] = l;
    mbar_arrive(bar + 8 * (C::bXFull + par));
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

// Epilogue warps (one warpgroup, thread = tile row r): per tile, combine the
// halves O = (O_0 2^(m_0 - M) + O_1 2^(m_1 - M)) / l, l = l_0 2^(m_0 - M) +
// l_1 2^(m_1 - M), lse = M + log l; stage the bf16 tile in swizzled shared
// memory and write it with one TMA tensor store.  Off the softmax warps' path:
// they hand over (m, l) and move on to the next tile.
template <int D>
__device__ int epi_warps(const Params& p, const Sched& sch, uint32_t base, uint8_t* gbase,
                         uint32_t tmem, int wq, int lane, const CUtensorMap* to) {
  using C = Cfg<D>;
  const AttnArgs& a = p.a;
  const uint32_t bar = base + C::oBar;
  const int r = wq * 32 + lane;
  const uint32_t trow = tmem + (static_cast<uint32_t>(wq * 32) << 16);
  const float* xs = reinterpret_cast<const float*>(gbase + C::oXSum);
  uint8_t* stg = gbase + C::oStg;
  const bool leader = r == 0;
  auto all_ok = [](bool ok) { return __all_sync(0xffffffffu, ok); };
  int tc = 0;
  for (int it = blockIdx.x; it < sch.count; it += gridDim.x) {
    const Item x = sched_item(p, sch, it);
    if (x.nch == 0) continue;
    const int64_t bh = static_cast<int64_t>(x.b) * a.heads + x.h;
    const int ob = tc % C::NOB, par = tc & 1;
    if (!all_ok(mbar_wait(bar + 8 * (C::bXFull + par), (tc >> 1) & 1))) return kErrXFull;
    const float m0 = xs[((par * 2 + 0) * 2 + 0) * 128 + r], l0 = xs[((par * 2 + 0) * 2 + 1) * 128 + r];
    const float m1 = xs[((par * 2 + 1) * 2 + 0) * 128 + r], l1 = xs[((par * 2 + 1) * 2 + 1) * 128 + r];
    mbar_arrive(bar + 8 * (C::bXFree + par));
    const float M = fmaxf(m0, m1);
    const float f0 = m0 == -INFINITY ? 0.f : ex2_approx(m0 - M);
    const float f1 = m1 == -INFINITY ? 0.f : ex2_approx(m1 - M);
    const float L = l0 * f0 + l1 * f1;
    const bool has = L > 0.f;  // padding rows and rows without a visible key: 0
    const float inv = has ? 1.f / L : 0.f;
    const float g0 = f0 * inv, g1 = f1 * inv;
#pragma unroll
    for (int h = 0; h < 2; ++h)
      if (!all_ok(mbar_wait(bar + 8 * (C::bOFull + h * C::NOB + ob), (tc / C::NOB) & 1)))
        return kErrOFull;
    tc_fence_after();
    if (leader) bulk_wait_read0();  // the previous tile's store is done with the staging
    named_barrier(2, 128);
#pragma unroll
    for (int j = 0; j < D / 32; ++j) {  // 32 output columns at a time
      float o0[32], o1[32];
      tmem_ld32(trow + C::tO(0, ob) + 32 * j, o0);
      tmem_ld32(trow + C::tO(1, ob) + 32 * j, o1);
      tmem_wait_ld();
      reg_fence(o0);
      reg_fence(o1);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        float w8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w8[i] = fmaf(o0[8 * v + i], g0, o1[8 * v + i] * g1);
        const int gc = 4 * j + v;  // 16-byte chunk index within the output row
        *reinterpret_cast<uint4*>(stg + (gc >> 3) * kSlab + r * 128 + (((gc & 7) ^ (r & 7)) << 4)) =
            make_uint4(pack_bf16(w8[0], w8[1]), pack_bf16(w8[2], w8[3]), pack_bf16(w8[4], w8[5]),
                       pack_bf16(w8[6], w8[7]));
      }
    }
    tc_fence_before();
    mbar_arrive(bar + 8 * (C::bOFree + 0 * C::NOB + ob));
    mbar_arrive(bar + 8 * (C::bOFree + 1 * C::NOB + ob));
    const int q = x.tile * kRows + r;
    if (q < a.n && a.lse) a.lse[bh * a.n + q] = has ? (M + log2f(L)) * kLn2 : -INFINITY;
    fence_proxy_async_smem();
    named_barrier(1, 128);  // the whole tile is staged
    if (leader) {
#pragma unroll
      for (int s = 0; s < D / 64; ++s)
        tma_store_3d(to, base + C::oStg + s * kSlab, s * 64, x.tile * kRows, static_cast<int>(bh));
      bulk_commit();
    }
    ++tc;
  }
  if (leader) bulk_wait_all0();  // the last tile's store has landed before the CTA exits
  return 0;
}

template <int D, bool kCausal>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to,
                       const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bar = base + C::oBar;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NQ; ++i) {
      mbar_init(bar + 8 * (C::bQFull + i), 1);
      mbar_init(bar + 8 * (C::bQFree + i), 1);
    }
    for (int i = 0; i < C::NKV; ++i) {
      mbar_init(bar + 8 * (C::bKFull + i), 1);
      mbar_init(bar + 8 * (C::bKFree + i), 1);
      mbar_init(bar + 8 * (C::bVFull + i), 1);
      mbar_init(bar + 8 * (C::bVFree + i), 1);
    }
    for (int i = 0; i < C::NSB; ++i) {
      mbar_init(bar + 8 * (C::bSFull + i), 1);
      mbar_init(bar + 8 * (C::bSFree + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar + 8 * (C::bXFull + i), 256);
      mbar_init(bar + 8 * (C::bXFree + i), 128);
    }
    for (int i = 0; i < 2 * C::NSB; ++i) {
      mbar_init(bar + 8 * (C::bPFull + i), 128);
      mbar_init(bar + 8 * (C::bPVDone + i), 1);
    }
    for (int i = 0; i < 2 * C::NOB; ++i) {
      mbar_init(bar + 8 * (C::bOFull + i), 1);
      mbar_init(bar + 8 * (C::bOFree + i), 128);
    }
    mbar_init(bar + 8 * C::bDone, 2);  // one commit per MMA-issuing thread
    fence_barrier_init();
  }
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tq);
      prefetch_tmap(&tk);
      prefetch_tmap(&tv);
      prefetch_tmap(&to);
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

  int err = 0;
  if (warp < 4) {
    regs_dec<C::kRegsCtl, kLaunchRegs>();
    if (warp == 0 && lane == 0) err = producer<D>(p, sch, base, &tq, &tk, &tv);
    if (warp == 1 && lane == 0) err = s_issuer<D>(p, sch, base, tmem);
    if (warp == 2 && lane == 0) err = pv_issuer<D>(p, sch, base, tmem);
    if (warp == 3 && lane == 0) err = v_producer<D>(p, sch, base, &tv);
  } else if (warp < 12) {
    regs_inc<C::kRegsSoft, kLaunchRegs>();
    err = softmax_warps<D, kCausal>(p, sch, base, gbase, tmem, warp & 3, (warp - 4) >> 2, lane);
  } else {
    regs_dec<C::kRegsEpi, kLaunchRegs>();
    err = epi_warps<D>(p, sch, base, gbase, tmem, warp & 3, lane, &to);
  }
  if (err) record_error(p.a.err, err);

  pdl_trigger();  // this CTA's work is issued: the next kernel may start launching
  __syncthreads();
  if (warp == 2 && lane == 0) mma_commit(bar + 8 * C::bDone);
  if (warp == 1) {
    if (lane == 0) {  // every tensor-core operation of this CTA has completed
      mma_commit(bar + 8 * C::bDone);
      if (!mbar_wait(bar + 8 * C::bDone, 0)) record_error(p.a.err, kErrDone);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D>
cudaError_t launch(const AttnArgs& a, cudaStream_t stream) {
  using C = Cfg<D>;
  const int64_t heads_total = static_cast<int64_t>(a.batch) * a.heads;
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_bf16_rows(&tq, a.q, D, a.n, heads_total, kRows) ||
      !make_tmap_bf16_rows(&tk, a.k, D, a.n, heads_total, kChunk) ||
      !make_tmap_bf16_rows(&tv, a.v, D, a.n, heads_total, kChunk) ||
      !make_tmap_bf16_rows(&to, a.o, D, a.n, heads_total, kRows))
    return cudaErrorInvalidValue;
  Params p;
  p.a = a;
  p.ntiles = (a.n + kRows - 1) / kRows;
  const int64_t items = heads_total * p.ntiles;
  if (items > (1ll << 30)) return cudaErrorInvalidValue;
  p.items = static_cast<int>(items);
  auto kernel = a.causal ? attn_fwd_tc_kernel<D, true> : attn_fwd_tc_kernel<D, false>;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(items < num_sms() ? items : num_sms());
  return launch_pdl(kernel, dim3(grid), dim3(kThreads), C::kSmem, stream, tq, tk, tv,
                    to, p);
}

}  // namespace

cudaError_t launch_attn_fwd_bf16_tc(const AttnArgs& a, cudaStream_t stream) {
  return a.d == 64 ? launch<64>(a, stream) : launch<128>(a, stream);
}

}  // namespace nb
