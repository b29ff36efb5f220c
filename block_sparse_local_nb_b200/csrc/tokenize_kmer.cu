// Fused 2-bit DNA k-mer tokenizer (NucleoByte page, section 1 "Token Blur",
// section 2 "Fused 2-Bit Tokenization", section 5 "Architecture Size").
//
// Each thread owns 32 consecutive bases (two 16-byte loads) plus a halo of the
// next 8 bytes (one 8-byte load that the neighbouring thread also reads; it is
// served from L1/L2, so HBM sees each byte once).  Per 32-bit word of 4 bytes:
//   code   = ((c >> 1) ^ (c >> 2)) & 3 per byte, which is 0, 1, 2, 3 for the
//            ASCII letters A, C, G, T;
//   valid  = the byte equals the letter of its code ('A','C','G','T' looked up
//            with one byte-permute), tested with an exact zero-byte test;
//   packed = the four codes of valid bytes, first byte in bits 7..6.
// The packed bytes of 24 consecutive bases form a 48-bit code register (first
// base most significant), so window j's ID is a funnel shift and a mask; a
// 24-bit mask of invalid bytes, OR-ed with itself shifted 1..k-1 places, flags
// the windows that contain one.  Outputs per thread: 32 uint16 IDs (four
// 16-byte stores) and 8 packed bytes (one 8-byte store).
//
// HBM bound: 1 byte read + 2 bytes (IDs) + 0.25 bytes (packed) written per base.
#include "nb_internal.h"

namespace nb {
namespace {

constexpr int kBases = 32;  // bases per thread

struct Word {
  uint32_t packed;  // four 2-bit codes, first byte in bits 7..6 (invalid -> 0)
  uint32_t bad;     // four invalid flags, first byte in bit 3
};

__device__ __forceinline__ Word classify(uint32_t w) {
  const uint32_t c = ((w >> 1) ^ (w >> 2)) & 0x03030303u;
  // byte-permute selector: nibble i = code of byte i, picking 'A','C','G','T'
  const uint32_t t = c | (c >> 4);  // codes of bytes 0, 1 at bits 0, 4; of bytes 2, 3 at 16, 20
  const uint32_t sel = (t & 0x33u) | ((t >> 8) & 0x3300u);
  const uint32_t x = __byte_perm(0x54474341u, 0u, sel) ^ w;  // zero byte <=> valid byte
  const uint32_t eq = ~(((x & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | x | 0x7F7F7F7Fu);  // 0x80 if zero
  const uint32_t cm = c & ((eq >> 7) * 3u);  // codes of invalid bytes cleared
  Word r;
  // one multiply gathers the four 2-bit codes into bits 31..24, byte 0 highest
  // (the shifted copies occupy disjoint bit ranges, so nothing carries)
  r.packed = (cm * 0x40100401u) >> 24;
  // likewise the four invalid flags (bit 7 of each byte) into bits 27..24
  r.bad = ((((~eq >> 7) & 0x01010101u) * 0x08040201u) >> 24) & 0xFu;
  return r;
}

// The 16 IDs of windows base0 + 16 h .. base0 + 16 h + 15 from words 4h .. 4h + 5.
template <int K>
__device__ __forceinline__ void window_ids(const Word (&wd)[10], int h, uint32_t (&out)[8]) {
  const uint32_t hi = (wd[4 * h].packed << 8) | wd[4 * h + 1].packed;  // bases 0..7 of the 24
  const uint32_t lo = (wd[4 * h + 2].packed << 24) | (wd[4 * h + 3].packed << 16) |
                      (wd[4 * h + 4].packed << 8) | wd[4 * h + 5].packed;  // bases 8..23
  const uint32_t B = (wd[4 * h].bad << 20) | (wd[4 * h + 1].bad << 16) | (wd[4 * h + 2].bad << 12) |
                     (wd[4 * h + 3].bad << 8) | (wd[4 * h + 4].bad << 4) | wd[4 * h + 5].bad;
  uint32_t W = B;  // bit p set <=> an invalid byte among bits p .. p + K - 1 of B
#pragma unroll
  for (int t = 1; t < K; ++t) W |= B >> t;
  constexpr uint32_t kMask = (1u << (2 * K)) - 1u;
  constexpr uint32_t kFlag = 1u << (2 * K);
  uint32_t id[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int sh = 24 - j - K;  // window j's last base sits at bits 2 sh + 1 .. 2 sh
    const uint32_t v = 2 * sh >= 32 ? (hi >> (2 * sh - 32)) : __funnelshift_r(lo, hi, 2 * sh);
    id[j] = ((W >> sh) & 1u) ? kFlag : (v & kMask);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) out[i] = id[2 * i] | (id[2 * i + 1] << 16);
}

template <int K, bool kAligned>
__global__ void __launch_bounds__(256) tokenize_kmer_kernel(const uint8_t* __restrict__ seq,
                                                            int64_t len, uint16_t* __restrict__ ids,
                                                            uint8_t* __restrict__ packed,
                                                            int64_t nchunks, bool ids_vec,
                                                            bool packed_vec) {
  __shared__ uint4 stage[256 * 4];
  pdl_trigger();
  pdl_wait();
  const int64_t nwin = len - K + 1;  // number of windows (may be <= 0)
  const int64_t npacked = (len + 3) >> 2;
  for (int64_t c = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; c < nchunks;
       c += (int64_t)gridDim.x * blockDim.x) {
    const int64_t base = c * kBases;
    uint32_t w[10];
    if (kAligned && base + kBases + 8 <= len) {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(seq + base));
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(seq + base + 16));
      const uint2 hl = __ldg(reinterpret_cast<const uint2*>(seq + base + 32));
      w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
      w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
      w[8] = hl.x; w[9] = hl.y;
    } else {
#pragma unroll
      for (int i = 0; i < 10; ++i) {
        uint32_t x = 0;
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) {
          const int64_t p = base + 4 * i + bb;
          const uint32_t byte = p < len ? __ldg(seq + p) : 0u;  // past the end: invalid, code 0
          x |= byte << (8 * bb);
        }
        w[i] = x;
      }
    }
    Word wd[10];
#pragma unroll
    for (int i = 0; i < 10; ++i) wd[i] = classify(w[i]);

    const int lane = threadIdx.x & 31;
    const int64_t wbase = base - lane * kBases;  // the warp's first window
    if (ids != nullptr && ids_vec && wbase + 32 * kBases <= nwin) {
      // whole warp in range: stage the 64-byte ID runs (16-byte chunks swizzled),
      // then write the warp's 2 KB span with coalesced 512-byte stores
      uint4* mine = stage + threadIdx.x * 4;
      const int sw = (lane >> 1) & 3;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t out[8];
        window_ids<K>(wd, h, out);
        mine[(2 * h) ^ sw] = make_uint4(out[0], out[1], out[2], out[3]);
        mine[(2 * h + 1) ^ sw] = make_uint4(out[4], out[5], out[6], out[7]);
      }
      __syncwarp();
      const uint4* wstage = stage + (threadIdx.x - lane) * 4;
      uint4* dst = reinterpret_cast<uint4*>(ids + wbase);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int c = 32 * r + lane, from = c >> 2;
        __stcs(dst + c, wstage[from * 4 + ((c & 3) ^ ((from >> 1) & 3))]);
      }
      __syncwarp();  // the staging is rewritten by the next iteration
    } else if (ids != nullptr) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t out[8];
        window_ids<K>(wd, h, out);
        const int64_t p0 = base + 16 * h;
        if (ids_vec && p0 + 16 <= nwin) {
          uint4* dst = reinterpret_cast<uint4*>(ids + p0);
          __stcs(dst, make_uint4(out[0], out[1], out[2], out[3]));
          __stcs(dst + 1, make_uint4(out[4], out[5], out[6], out[7]));
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (p0 + j < nwin) ids[p0 + j] = static_cast<uint16_t>(out[j >> 1] >> (16 * (j & 1)));
        }
      }
    }
    if (packed != nullptr) {
      const int64_t pb = c * (kBases / 4);
      const uint32_t lo = wd[0].packed | (wd[1].packed << 8) | (wd[2].packed << 16) |
                          (wd[3].packed << 24);
      const uint32_t hi = wd[4].packed | (wd[5].packed << 8) | (wd[6].packed << 16) |
                          (wd[7].packed << 24);
      if (packed_vec && pb + 8 <= npacked) {
        __stcs(reinterpret_cast<uint2*>(packed + pb), make_uint2(lo, hi));
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (pb + i < npacked) packed[pb + i] = static_cast<uint8_t>(wd[i].packed);
      }
    }
  }
}

template <int K>
cudaError_t launch_k(const uint8_t* seq, int64_t len, uint16_t* ids, uint8_t* packed,
                     int64_t nchunks, unsigned blocks, bool aligned, bool ids_vec, bool packed_vec,
                     cudaStream_t stream) {
  if (aligned)
    return launch_pdl(tokenize_kmer_kernel<K, true>, dim3(blocks), dim3(256), 0, stream, seq, len,
                      ids, packed, nchunks, ids_vec, packed_vec);
  return launch_pdl(tokenize_kmer_kernel<K, false>, dim3(blocks), dim3(256), 0, stream, seq, len,
                    ids, packed, nchunks, ids_vec, packed_vec);
}

// Batch to model input IDs: thread = 32 consecutive windows of one sequence
// (blockIdx.y).  Model ID = raw window ID + 1, so the flag 4^K becomes 4^K + 1;
// windows at or past the sequence's window count (or n_pad) are padding (0).
template <int K>
__global__ void __launch_bounds__(128) tokenize_batch_kernel(const uint8_t* __restrict__ seqs,
                                                             const int64_t* __restrict__ offsets,
                                                             int64_t* __restrict__ ids,
                                                             int32_t* __restrict__ lengths,
                                                             int n_pad) {
  // per thread: its 32 IDs (256 bytes) staged with a 16-byte-chunk swizzle, then
  // each warp writes its contiguous 8 KB span with 512-byte coalesced stores
  __shared__ uint4 stage[128 * 16];
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t s0 = offsets[b];
  const int64_t nbases = max(offsets[b + 1] - s0, (int64_t)0);
  const int len = static_cast<int>(min(max(nbases - K + 1, (int64_t)0), (int64_t)n_pad));
  if (lengths != nullptr && blockIdx.x == 0 && threadIdx.x == 0) lengths[b] = len;
  const int t0 = (blockIdx.x * blockDim.x + threadIdx.x) * kBases;  // first window
  uint4* mine = stage + threadIdx.x * 16;
  if (t0 < n_pad && t0 >= len) {  // all padding
#pragma unroll
    for (int j = 0; j < 16; ++j) mine[j ^ (lane & 15)] = make_uint4(0, 0, 0, 0);
  } else if (t0 < n_pad) {
    // bases t0 .. t0 + 39 of this sequence (past its end: 0, an invalid byte)
    const uint8_t* src = seqs + s0 + t0;
    const int64_t avail = nbases - t0;
    uint32_t w[10];
#pragma unroll
    for (int i = 0; i < 10; ++i) {
      uint32_t x = 0;
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) {
        const int p = 4 * i + bb;
        const uint32_t byte = p < avail ? __ldg(src + p) : 0u;
        x |= byte << (8 * bb);
      }
      w[i] = x;
    }
    Word wd[10];
#pragma unroll
    for (int i = 0; i < 10; ++i) wd[i] = classify(w[i]);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t out[8];
      window_ids<K>(wd, h, out);
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        const int t = t0 + 16 * h + j;
        const uint32_t r0 = out[j >> 1] & 0xFFFFu, r1 = out[j >> 1] >> 16;
        const uint32_t m0 = t < len ? r0 + 1u : 0u, m1 = t + 1 < len ? r1 + 1u : 0u;
        mine[(8 * h + (j >> 1)) ^ (lane & 15)] = make_uint4(m0, 0u, m1, 0u);
      }
    }
  }
  __syncwarp();
  const int wt0 = t0 - lane * kBases;  // the warp's first window
  const int count = min(32 * kBases, n_pad - wt0) / 2;  // 16-byte chunks of the warp's span
  uint4* dst = reinterpret_cast<uint4*>(ids + static_cast<int64_t>(b) * n_pad + wt0);
  const uint4* wstage = stage + warp * 32 * 16;
  for (int c = lane; c < count; c += 32) {
    const int from = c >> 4;  // the lane that produced chunk c
    __stcs(dst + c, wstage[from * 16 + ((c & 15) ^ (from & 15))]);
  }
}

template <int K>
cudaError_t launch_batch_k(const uint8_t* seqs, const int64_t* offsets, int batch, int64_t* ids,
                           int32_t* lengths, int n_pad, cudaStream_t stream) {
  const int chunks = n_pad / kBases;
  const unsigned gx = static_cast<unsigned>(chunks > 0 ? (chunks + 127) / 128 : 1);
  return launch_pdl(tokenize_batch_kernel<K>, dim3(gx, static_cast<unsigned>(batch)), dim3(128), 0,
                    stream, seqs, offsets, ids, lengths, n_pad);
}

}  // namespace

cudaError_t launch_tokenize_batch(const uint8_t* seqs, const int64_t* offsets, int batch, int k,
                                  int64_t* ids, int32_t* lengths, int n_pad, cudaStream_t stream) {
  switch (k) {
    case 1: return launch_batch_k<1>(seqs, offsets, batch, ids, lengths, n_pad, stream);
    case 2: return launch_batch_k<2>(seqs, offsets, batch, ids, lengths, n_pad, stream);
    case 3: return launch_batch_k<3>(seqs, offsets, batch, ids, lengths, n_pad, stream);
    case 4: return launch_batch_k<4>(seqs, offsets, batch, ids, lengths, n_pad, stream);
    case 5: return launch_batch_k<5>(seqs, offsets, batch, ids, lengths, n_pad, stream);
    case 6: return launch_batch_k<6>(seqs, offsets, batch, ids, lengths, n_pad, stream);
    default: return launch_batch_k<7>(seqs, offsets, batch, ids, lengths, n_pad, stream);
  }
}

cudaError_t launch_tokenize_kmer(const uint8_t* seq, int64_t len, uint16_t* ids, uint8_t* packed,
                                 int k, cudaStream_t stream) {
  const int64_t nchunks = (len + kBases - 1) / kBases;
  if (nchunks == 0 || (ids == nullptr && packed == nullptr)) return cudaSuccess;
  const int threads = 256;
  int64_t blocks = (nchunks + threads - 1) / threads;
  // a few waves of blocks that loop over the rest (measured: fewer, longer-lived
  // blocks beat one short block per 8 KB of input)
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  if (blocks > cap) blocks = cap;
  const bool aligned = (reinterpret_cast<uintptr_t>(seq) & 15u) == 0;
  const bool ids_vec = (reinterpret_cast<uintptr_t>(ids) & 15u) == 0;
  const bool packed_vec = (reinterpret_cast<uintptr_t>(packed) & 7u) == 0;
  const unsigned b = static_cast<unsigned>(blocks);
  switch (k) {
    case 1: return launch_k<1>(seq, len, ids, packed, nchunks, b, aligned, ids_vec, packed_vec, stream);
    case 2: return launch_k<2>(seq, len, ids, packed, nchunks, b, aligned, ids_vec, packed_vec, stream);
    case 3: return launch_k<3>(seq, len, ids, packed, nchunks, b, aligned, ids_vec, packed_vec, stream);
    case 4: return launch_k<4>(seq, len, ids, packed, nchunks, b, aligned, ids_vec, packed_vec, stream);
    case 5: return launch_k<5>(seq, len, ids, packed, nchunks, b, aligned, ids_vec, packed_vec, stream);
    case 6: return launch_k<6>(seq, len, ids, packed, nchunks, b, aligned, ids_vec, packed_vec, stream);
    default: return launch_k<7>(seq, len, ids, packed, nchunks, b, aligned, ids_vec, packed_vec, stream);
  }
}

}  // namespace nb
