// Fused 2-bit DNA k-mer tokenizer (NucleoByte page, section 1 "Token Blur",
// section 2 "Fused 2-Bit Tokenization", section 5 "Architecture Size").
//
// Each thread owns 16 consecutive bases (one 16-byte load) plus a halo of the
// next 8 bytes (one 8-byte load that the neighbouring thread also reads; it is
// served from L1/L2, so HBM sees each byte once).  Per 32-bit word the four
// bytes are classified with byte-SIMD compares and turned into 2-bit codes
// with shifts: for the ASCII letters A, C, G, T ((c >> 1) ^ (c >> 2)) & 3 is
// 0, 1, 2, 3.  The 24 codes go into one 48-bit register, first base most
// significant, so window j's ID is a shift and a mask; a 24-bit mask of
// invalid bytes flags windows that contain one.  Outputs: 16 uint16 IDs (two
// 16-byte stores) and 4 packed bytes (one 4-byte store) per thread.
//
// HBM bound: 1 byte read + 2 bytes (IDs) + 0.25 bytes (packed) written per base.
#include "nb_internal.h"

namespace nb {
namespace {

constexpr uint32_t kRep = 0x01010101u;

struct Word {
  uint32_t packed;  // four 2-bit codes, first byte in bits 7..6 (invalid -> 0)
  uint32_t bad;     // four invalid flags, first byte in bit 3
};

__device__ __forceinline__ Word classify(uint32_t w) {
  uint32_t ok = __vcmpeq4(w, 'A' * kRep) | __vcmpeq4(w, 'C' * kRep) | __vcmpeq4(w, 'G' * kRep) |
                __vcmpeq4(w, 'T' * kRep);
  uint32_t c = ((w >> 1) ^ (w >> 2)) & 0x03030303u & ok;
  Word r;
  r.packed = ((c & 3u) << 6) | (((c >> 8) & 3u) << 4) | (((c >> 16) & 3u) << 2) | (c >> 24);
  uint32_t inv = ~ok;
  r.bad = (((inv >> 7) & 1u) << 3) | (((inv >> 15) & 1u) << 2) | (((inv >> 23) & 1u) << 1) |
          (inv >> 31);
  return r;
}

template <bool kAligned>
__global__ void __launch_bounds__(256) tokenize_kmer_kernel(const uint8_t* __restrict__ seq,
                                                            int64_t len, uint16_t* __restrict__ ids,
                                                            uint8_t* __restrict__ packed, int k,
                                                            int64_t nchunks, bool ids_vec,
                                                            bool packed_vec) {
  const int64_t nwin = len - k + 1;  // number of windows (may be <= 0)
  const int64_t npacked = (len + 3) >> 2;
  const uint32_t idmask = (1u << (2 * k)) - 1u;
  const uint32_t badmask = (1u << k) - 1u;
  const uint16_t flag = static_cast<uint16_t>(1u << (2 * k));
  for (int64_t c = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; c < nchunks;
       c += (int64_t)gridDim.x * blockDim.x) {
    const int64_t base = c * 16;
    uint32_t w[6];
    if (kAligned && base + 24 <= len) {
      uint4 a = __ldg(reinterpret_cast<const uint4*>(seq + base));
      uint2 h = __ldg(reinterpret_cast<const uint2*>(seq + base + 16));
      w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = h.x; w[5] = h.y;
    } else {
#pragma unroll
      for (int i = 0; i < 6; ++i) {
        uint32_t x = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          int64_t p = base + 4 * i + b;
          uint32_t byte = p < len ? __ldg(seq + p) : 0u;  // past the end: invalid, code 0
          x |= byte << (8 * b);
        }
        w[i] = x;
      }
    }
    uint64_t codes = 0;
    uint32_t bad = 0;
    uint32_t pk[4];
#pragma unroll
    for (int i = 0; i < 6; ++i) {
      Word r = classify(w[i]);
      codes = (codes << 8) | r.packed;
      bad = (bad << 4) | r.bad;
      if (i < 4) pk[i] = r.packed;
    }
    // base i of the 24 sits at bits 2*(23-i)+1..2*(23-i); window j covers bases j..j+k-1
    if (ids != nullptr) {
      uint32_t out[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int sh = 24 - j - k;
        uint32_t id = static_cast<uint32_t>(codes >> (2 * sh)) & idmask;
        out[j] = ((bad >> sh) & badmask) ? flag : id;
      }
      if (ids_vec && base + 16 <= nwin) {
        uint4 lo = make_uint4(out[0] | (out[1] << 16), out[2] | (out[3] << 16),
                              out[4] | (out[5] << 16), out[6] | (out[7] << 16));
        uint4 hi = make_uint4(out[8] | (out[9] << 16), out[10] | (out[11] << 16),
                              out[12] | (out[13] << 16), out[14] | (out[15] << 16));
        uint4* dst = reinterpret_cast<uint4*>(ids + base);
        __stcs(dst, lo);
        __stcs(dst + 1, hi);
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (base + j < nwin) ids[base + j] = static_cast<uint16_t>(out[j]);
      }
    }
    if (packed != nullptr) {
      const int64_t pb = c * 4;
      if (packed_vec && pb + 4 <= npacked) {
        __stcs(reinterpret_cast<unsigned int*>(packed + pb),
               pk[0] | (pk[1] << 8) | (pk[2] << 16) | (pk[3] << 24));
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (pb + i < npacked) packed[pb + i] = static_cast<uint8_t>(pk[i]);
      }
    }
  }
}

}  // namespace

cudaError_t launch_tokenize_kmer(const uint8_t* seq, int64_t len, uint16_t* ids, uint8_t* packed,
                                 int k, cudaStream_t stream) {
  const int64_t nchunks = (len + 15) / 16;
  if (nchunks == 0 || (ids == nullptr && packed == nullptr)) return cudaSuccess;
  const int threads = 256;
  int64_t blocks = (nchunks + threads - 1) / threads;
  if (blocks > (1 << 30)) blocks = 1 << 30;  // grid-stride loop covers the rest
  const bool aligned = (reinterpret_cast<uintptr_t>(seq) & 15u) == 0;
  const bool ids_vec = (reinterpret_cast<uintptr_t>(ids) & 15u) == 0;
  const bool packed_vec = (reinterpret_cast<uintptr_t>(packed) & 3u) == 0;
  if (aligned)
    tokenize_kmer_kernel<true><<<(unsigned)blocks, threads, 0, stream>>>(
        seq, len, ids, packed, k, nchunks, ids_vec, packed_vec);
  else
    tokenize_kmer_kernel<false><<<(unsigned)blocks, threads, 0, stream>>>(
        seq, len, ids, packed, k, nchunks, ids_vec, packed_vec);
  return cudaGetLastError();
}

}  // namespace nb
