// Fused 2-bit DNA k-mer tokenizer (NucleoByte page, section 1 "Token Blur",
// section 2 "Fused 2-Bit Tokenization", section 5 "Architecture Size").
//
// A thread turns 32 consecutive bases plus the next 8 (the windows' halo)
// into 32 IDs and 8 packed bytes.  Per 32-bit word of 4 bytes:
//   code   = ((c >> 1) ^ (c >> 2)) & 3 per byte, which is 0, 1, 2, 3 for the
//            ASCII letters A, C, G, T;
//   valid  = the byte equals the letter of its code ('A','C','G','T' looked up
//            with one byte-permute), tested with an exact zero-byte test;
//   packed = the four codes of valid bytes, first byte in bits 7..6.
// The packed bytes of 24 consecutive bases form a 48-bit code register (first
// base most significant), so window j's ID is a funnel shift and a mask; a
// 24-bit mask of invalid bytes, OR-ed with itself shifted 1..k-1 places, flags
// the windows that contain one.
//
// Data movement: the sequence is cut into tiles of 8192 bases that the
// bulk-copy (TMA) engine loads into shared memory, several tiles ahead per
// block; the IDs and packed bytes of a tile are assembled in shared memory
// and leave with two bulk stores (see tokenize_kmer_kernel).  The tail, and
// buffers that are not 16-byte aligned, are handled per thread with direct
// loads and stores (chunk_direct).
//
// HBM bound: 1 byte read + 2 bytes (IDs) + 0.25 bytes (packed) written per base.
#include "nb_internal.h"
#include "sm100.cuh"

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

// One chunk c of 32 bases handled by one thread on its own: bounds-checked
// loads (16-byte loads when `seq_vec` and inside), IDs and packed bytes
// written directly.  Serves the sequence's tail and buffers that are not
// 16-byte aligned.
template <int K>
__device__ __forceinline__ void chunk_direct(const uint8_t* __restrict__ seq, int64_t len,
                                             uint16_t* __restrict__ ids,
                                             uint8_t* __restrict__ packed, int64_t c, bool seq_vec,
                                             bool ids_vec, bool packed_vec) {
  const int64_t nwin = len - K + 1;  // number of windows (may be <= 0)
  const int64_t npacked = (len + 3) >> 2;
  const int64_t base = c * kBases;
  uint32_t w[10];
  if (seq_vec && base + kBases + 8 <= len) {
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

// Tiles of 8192 bases moved by the bulk-copy (TMA) engine: each block keeps
// kStagesIn tiles of input in flight (one bulk load of 8192 + 16 bytes each,
// the 16 bytes being the next tile's first bases, which the last windows
// read), its 256 threads turn one tile into 16 KB of IDs and 2 KB of packed
// bytes in shared memory, and one thread writes them back with two bulk
// stores, double-buffered.  The bytes in flight per SM, not the thread count,
// then keep HBM busy.  Tiles whose input would reach past the sequence, and
// every chunk when a buffer is not 16-byte aligned, go through chunk_direct.
constexpr int kTileBases = 256 * kBases;           // 8192
constexpr int kInBytes = kTileBases + 16;          // + the halo, a multiple of 16
constexpr int kStagesIn = 4;
constexpr int kIdBytes = kTileBases * 2;           // 16 KB
constexpr int kOutBytes = kIdBytes + kTileBases / 4;  // + 2 KB packed
constexpr int kTokSmem = kStagesIn * kInBytes + 2 * kOutBytes + kStagesIn * 8;

__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                   reinterpret_cast<uint64_t>(dst)),
               "r"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_wait_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

template <int K>
__global__ void __launch_bounds__(256, 3) tokenize_kmer_kernel(const uint8_t* __restrict__ seq,
                                                               int64_t len, uint16_t* __restrict__ ids,
                                                               uint8_t* __restrict__ packed,
                                                               int64_t ntiles, int64_t nchunks,
                                                               bool seq_vec, bool ids_vec,
                                                               bool packed_vec, int* err) {
  using namespace sm100;
  extern __shared__ __align__(128) uint8_t tsm[];
  const uint32_t sin = smem_u32(tsm);                // input stages
  const uint32_t sout = sin + kStagesIn * kInBytes;  // two output buffers
  const uint32_t bar = sout + 2 * kOutBytes;         // kStagesIn mbarriers
  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int i = 0; i < kStagesIn; ++i) mbar_init(bar + 8 * i, 1);
    fence_barrier_init();
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();
  // this block's tiles: blockIdx.x + k gridDim.x, k < mine
  const int64_t mine = ntiles > blockIdx.x ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  auto load = [&](int64_t k) {
    const int st = static_cast<int>(k % kStagesIn);
    const int64_t t = blockIdx.x + k * gridDim.x;
    mbar_arrive_expect_tx(bar + 8 * st, kInBytes);
    bulk_load(sin + st * kInBytes, seq + t * kTileBases, kInBytes, bar + 8 * st);
  };
  if (tid == 0)
    for (int64_t k = 0; k < mine && k < kStagesIn; ++k) load(k);
  for (int64_t k = 0; k < mine; ++k) {
    const int64_t t = blockIdx.x + k * gridDim.x;
    const int si = static_cast<int>(k % kStagesIn), so = static_cast<int>(k & 1);
    if (tid == 0) bulk_wait_read1();  // the store of tile k - 2 has read output buffer `so`
    const bool ok = mbar_wait(bar + 8 * si, static_cast<uint32_t>((k / kStagesIn) & 1));
    if (!__syncthreads_and(ok)) {  // block-uniform: every thread gives up together
      if (tid == 0) record_error(err, 0x51);
      break;
    }
    // this thread's 32 bases and the 8 after them
    const uint8_t* src = tsm + si * kInBytes + kBases * tid;
    const uint4 a = *reinterpret_cast<const uint4*>(src);
    const uint4 b = *reinterpret_cast<const uint4*>(src + 16);
    const uint2 hl = *reinterpret_cast<const uint2*>(src + 32);
    const uint32_t w[10] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w, hl.x, hl.y};
    Word wd[10];
#pragma unroll
    for (int i = 0; i < 10; ++i) wd[i] = classify(w[i]);
    uint8_t* out = tsm + kStagesIn * kInBytes + so * kOutBytes;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t o[8];
      window_ids<K>(wd, h, o);
      uint4* dst = reinterpret_cast<uint4*>(out + 64 * tid + 32 * h);
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
    *reinterpret_cast<uint2*>(out + kIdBytes + 8 * tid) =
        make_uint2(wd[0].packed | (wd[1].packed << 8) | (wd[2].packed << 16) | (wd[3].packed << 24),
                   wd[4].packed | (wd[5].packed << 8) | (wd[6].packed << 16) | (wd[7].packed << 24));
    fence_proxy_async_smem();
    __syncthreads();  // input stage si read, output buffer so written
    if (tid == 0) {
      if (ids != nullptr) bulk_store(ids + t * kTileBases, sout + so * kOutBytes, kIdBytes);
      if (packed != nullptr)
        bulk_store(packed + t * (kTileBases / 4), sout + so * kOutBytes + kIdBytes, kTileBases / 4);
      bulk_commit();
      if (k + kStagesIn < mine) load(k + kStagesIn);
    }
  }
  if (tid == 0) bulk_wait_all0();  // the stores have landed (and read shared memory) before exit
  // the tail (and everything when a buffer is not 16-byte aligned)
  for (int64_t c = ntiles * 256 + blockIdx.x * (int64_t)blockDim.x + tid; c < nchunks;
       c += (int64_t)gridDim.x * blockDim.x)
    chunk_direct<K>(seq, len, ids, packed, c, seq_vec, ids_vec, packed_vec);
}

template <int K>
cudaError_t launch_k(const uint8_t* seq, int64_t len, uint16_t* ids, uint8_t* packed,
                     int64_t ntiles, int64_t nchunks, unsigned blocks, bool seq_vec, bool ids_vec,
                     bool packed_vec, int* err, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(tokenize_kmer_kernel<K>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kTokSmem);
  if (e != cudaSuccess) return e;
  return launch_pdl(tokenize_kmer_kernel<K>, dim3(blocks), dim3(256), kTokSmem, stream, seq, len,
                    ids, packed, ntiles, nchunks, seq_vec, ids_vec, packed_vec, err);
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
                                 int k, int* err, cudaStream_t stream) {
  const int64_t nchunks = (len + kBases - 1) / kBases;
  if (nchunks == 0 || (ids == nullptr && packed == nullptr)) return cudaSuccess;
  const bool seq_vec = (reinterpret_cast<uintptr_t>(seq) & 15u) == 0;
  const bool ids_vec = (reinterpret_cast<uintptr_t>(ids) & 15u) == 0;
  const bool packed_vec = (reinterpret_cast<uintptr_t>(packed) & 15u) == 0;
  // whole tiles whose input, halo included, lies inside the sequence; all
  // their windows exist, so their IDs fill whole 16 KB runs
  int64_t ntiles = len >= 16 ? (len - 16) / kTileBases : 0;
  if (!(seq_vec && (ids == nullptr || ids_vec) && (packed == nullptr || packed_vec))) ntiles = 0;
  // three blocks per SM (shared-memory bound), each walking its tiles; at least
  // enough blocks that the tail's chunks are one per thread
  const int64_t tail_blocks = (nchunks - ntiles * 256 + 255) / 256;
  int64_t blocks = static_cast<int64_t>(num_sms()) * 3;
  if (ntiles < blocks) blocks = ntiles > tail_blocks ? ntiles : tail_blocks;
  if (blocks < 1) blocks = 1;
  const unsigned b = static_cast<unsigned>(blocks);
  switch (k) {
    case 1: return launch_k<1>(seq, len, ids, packed, ntiles, nchunks, b, seq_vec, ids_vec, packed_vec, err, stream);
    case 2: return launch_k<2>(seq, len, ids, packed, ntiles, nchunks, b, seq_vec, ids_vec, packed_vec, err, stream);
    case 3: return launch_k<3>(seq, len, ids, packed, ntiles, nchunks, b, seq_vec, ids_vec, packed_vec, err, stream);
    case 4: return launch_k<4>(seq, len, ids, packed, ntiles, nchunks, b, seq_vec, ids_vec, packed_vec, err, stream);
    case 5: return launch_k<5>(seq, len, ids, packed, ntiles, nchunks, b, seq_vec, ids_vec, packed_vec, err, stream);
    case 6: return launch_k<6>(seq, len, ids, packed, ntiles, nchunks, b, seq_vec, ids_vec, packed_vec, err, stream);
    default: return launch_k<7>(seq, len, ids, packed, ntiles, nchunks, b, seq_vec, ids_vec, packed_vec, err, stream);
  }
}

}  // namespace nb
