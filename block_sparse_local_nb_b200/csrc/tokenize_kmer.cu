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
  const uint32_t sel = (c & 0x3u) | ((c >> 4) & 0x30u) | ((c >> 8) & 0x300u) | ((c >> 12) & 0x3000u);
  const uint32_t x = __byte_perm(0x54474341u, 0u, sel) ^ w;  // zero byte <=> valid byte
  const uint32_t eq = ~(((x & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | x | 0x7F7F7F7Fu);  // 0x80 if zero
  const uint32_t cm = c & ((eq >> 7) * 3u);  // codes of invalid bytes cleared
  Word r;
  r.packed = ((cm << 6) | (cm >> 4) | (cm >> 14) | (cm >> 24)) & 0xFFu;
  const uint32_t inv = ~eq & 0x80808080u;
  r.bad = ((inv >> 4) & 8u) | ((inv >> 13) & 4u) | ((inv >> 22) & 2u) | (inv >> 31);
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

    if (ids != nullptr) {
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

}  // namespace

cudaError_t launch_tokenize_kmer(const uint8_t* seq, int64_t len, uint16_t* ids, uint8_t* packed,
                                 int k, cudaStream_t stream) {
  const int64_t nchunks = (len + kBases - 1) / kBases;
  if (nchunks == 0 || (ids == nullptr && packed == nullptr)) return cudaSuccess;
  const int threads = 256;
  int64_t blocks = (nchunks + threads - 1) / threads;
  if (blocks > (1 << 30)) blocks = 1 << 30;  // grid-stride loop covers the rest
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
