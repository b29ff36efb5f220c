// Forward + backward on host-resident tensors (nb_attn_fwd_bwd_host): the
// problem is cut into chunks and every chunk goes through three stages on
// three streams: copy-in (q, k, v, dO), compute (nb_attn_fwd then nb_attn_bwd
// on the caller's stream) and copy-out (O, lse, dQ, dK, dV).  Chunk i + 1 is
// copied in while chunk i computes and chunk i - 1 is copied out, so the host
// link carries both directions at once and the kernels hide behind the
// copies.  The device side holds kSlots chunks at a time in the caller's
// workspace.
//
// A chunk is either a group of whole (batch, head) slices, which attention
// treats independently, or - when there are too few slices to fill the
// pipeline - a window of one slice's sequence: the blocks [lo, hi) that the
// chunk owns plus 2R blocks of context on each side (clipped to the
// sequence), computed as a sequence of its own.  On such a window the
// forward's O and log-sum-exp are exact on every query block whose band lies
// inside it (R blocks from either cut), hence on its owned blocks; the
// backward, given those, is exact for dQ there and for dK and dV on blocks
// whose queries' bands lie inside it (2R from either cut), again the owned
// blocks.  (NucleoByte page, section 3: the band |i - j| <= R bounds which
// blocks a block's results depend on.)  Only the owned rows are copied back.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "../../include/nb.h"
#include "nb_internal.h"

namespace {

constexpr int kSlots = 3;        // chunks resident on the device at once
constexpr int64_t kChunks = 32;  // aim: this many chunks (pipeline depth)

struct Chunk {
  int b0, nbr, h0, nh;  // batch rows [b0, b0 + nbr) x heads [h0, h0 + nh)
  int a, w;             // device window: blocks [a, a + w) of each slice (whole: 0, nb)
  int lo, hi;           // blocks [lo, hi) copied back (whole: 0, nb)
  bool window;          // one slice cut along the sequence
};

struct Plan {
  std::vector<Chunk> chunks;
  int slots;
  int64_t max_rows;   // device rows of the largest chunk
  size_t len_bytes;   // device copy of lengths + one window length per chunk
  size_t tensor;      // one [max_rows x d] bf16 buffer
  size_t slot_bytes;  // one chunk's tensors + backward workspace
  size_t ws_off;      // offset of the backward workspace inside a slot
};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// cuMemsetD32Async, looked up at run time (the library does not link libcuda):
// writes a window's length into the workspace by value, in stream order, with
// no host staging buffer.
PFN_cuMemsetD32Async_v3020 g_memset32 = nullptr;
std::once_flag g_memset32_once;

PFN_cuMemsetD32Async_v3020 memset32_fn() {
  std::call_once(g_memset32_once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuMemsetD32Async", &p, 3020, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_memset32 = reinterpret_cast<PFN_cuMemsetD32Async_v3020>(p);
  });
  return g_memset32;
}

Plan make_plan(int batch, int heads, int n, int d, int R) {
  Plan p{};
  const int nb = n / NB_BLOCK;
  const int64_t units = static_cast<int64_t>(batch) * heads;
  if (units >= kChunks) {  // groups of whole slices
    const int64_t target = (units + kChunks - 1) / kChunks;
    if (target >= heads) {
      const int rows = static_cast<int>(target / heads);
      for (int b = 0; b < batch; b += rows)
        p.chunks.push_back({b, std::min(rows, batch - b), 0, heads, 0, nb, 0, nb, false});
    } else {
      const int hp = static_cast<int>(target);
      for (int b = 0; b < batch; ++b)
        for (int h = 0; h < heads; h += hp)
          p.chunks.push_back({b, 1, h, std::min(hp, heads - h), 0, nb, 0, nb, false});
    }
  } else {  // each slice in `parts` windows, each owning at least max(8, 4R) blocks
    const int64_t want = (kChunks + units - 1) / units;
    const int64_t min_own = std::max<int64_t>(8, 4 * static_cast<int64_t>(R));
    const int64_t parts = std::max<int64_t>(1, std::min<int64_t>(want, nb / min_own));
    const int own = static_cast<int>((nb + parts - 1) / parts);
    const int64_t halo = 2 * static_cast<int64_t>(R);
    for (int b = 0; b < batch; ++b)
      for (int h = 0; h < heads; ++h)
        for (int lo = 0; lo < nb; lo += own) {
          const int hi = std::min(nb, lo + own);
          const int a = static_cast<int>(std::max<int64_t>(0, lo - halo));
          const int e = static_cast<int>(std::min<int64_t>(nb, hi + halo));
          p.chunks.push_back({b, 1, h, 1, a, e - a, lo, hi, parts > 1});
        }
  }
  p.max_rows = 0;
  for (const Chunk& c : p.chunks)
    p.max_rows = std::max<int64_t>(p.max_rows,
                                   static_cast<int64_t>(c.nbr) * c.nh * c.w * NB_BLOCK);
  p.slots = static_cast<int>(std::min<size_t>(p.chunks.size(), kSlots));
  p.len_bytes = up256((static_cast<size_t>(batch) + p.chunks.size()) * 4);
  p.tensor = up256(static_cast<size_t>(p.max_rows) * d * 2);
  const size_t lse = up256(static_cast<size_t>(p.max_rows) * 4);
  p.ws_off = 8 * p.tensor + lse;
  p.slot_bytes = p.ws_off + up256(nb::bwd_workspace_bytes(p.max_rows, d));
  return p;
}

bool shape_ok(int batch, int heads, int n, int d, int dtype) {
  // the same shape rules as nb_attn_bwd (which the compute stage calls)
  return nb_attn_bwd_workspace_size(batch, heads, n, d, dtype) > 0 && dtype == NB_BF16;
}

}  // namespace

extern "C" {

size_t nb_attn_fwd_bwd_host_workspace_size(int batch, int heads, int n, int d, int R, int dtype) {
  if (R < 0 || !shape_ok(batch, heads, n, d, dtype)) return 0;
  const Plan p = make_plan(batch, heads, n, d, R);
  return p.len_bytes + static_cast<size_t>(p.slots) * p.slot_bytes;
}

nb_status nb_attn_fwd_bwd_host(const void* q, const void* k, const void* v, const void* dout,
                               const int32_t* lengths, void* o, float* lse, void* dq, void* dk,
                               void* dv, void* workspace, size_t workspace_bytes, int batch,
                               int heads, int n, int d, int R, int dtype, int causal,
                               void* stream) {
  if (batch < 0 || heads < 0 || n < 0 || R < 0 || (n % NB_BLOCK) != 0)
    return NB_ERR_INVALID_ARG;
  if (static_cast<int64_t>(batch) * heads * n == 0) return NB_OK;
  if (dtype != NB_BF16) return dtype == NB_F32 ? NB_ERR_UNSUPPORTED : NB_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return NB_ERR_UNSUPPORTED;
  if (!shape_ok(batch, heads, n, d, dtype)) return NB_ERR_INVALID_ARG;
  if (!q || !k || !v || !dout || !o || !dq || !dk || !dv) return NB_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_bytes < nb_attn_fwd_bwd_host_workspace_size(batch, heads, n, d, R, dtype))
    return NB_ERR_WORKSPACE;
  const nb_status dev_st = nb::device_check();
  if (dev_st != NB_OK) return dev_st;

  const Plan p = make_plan(batch, heads, n, d, R);
  const int64_t nchunks = static_cast<int64_t>(p.chunks.size());
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  // device lengths: the caller's [batch], then one window length per chunk
  int32_t* len_dev = reinterpret_cast<int32_t*>(ws);
  PFN_cuMemsetD32Async_v3020 memset32 = nullptr;
  if (lengths && p.chunks.front().window) {
    memset32 = memset32_fn();
    if (!memset32) return NB_ERR_CUDA;
  }
  const size_t row = static_cast<size_t>(d) * 2;  // bytes of one bf16 row

  cudaStream_t s_in = nullptr, s_out = nullptr;
  std::vector<cudaEvent_t> ev;  // [start] + per chunk [in, compute, out]
  nb_status st = NB_OK;
  auto fail = [&](cudaError_t e) {
    if (e != cudaSuccess && st == NB_OK) st = NB_ERR_CUDA;
    return e != cudaSuccess;
  };
  if (fail(cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking)) ||
      fail(cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking))) {
    if (s_in) cudaStreamDestroy(s_in);
    return st;
  }
  ev.resize(1 + 3 * nchunks, nullptr);
  for (auto& e : ev)
    if (fail(cudaEventCreateWithFlags(&e, cudaEventDisableTiming))) break;

  auto ev_in = [&](int64_t c) { return ev[1 + 3 * c]; };
  auto ev_comp = [&](int64_t c) { return ev[2 + 3 * c]; };
  auto ev_out = [&](int64_t c) { return ev[3 + 3 * c]; };
  if (st == NB_OK) {
    // the copies start after the caller's earlier work on `stream` (which may
    // still use the workspace)
    fail(cudaEventRecord(ev[0], cs));
    fail(cudaStreamWaitEvent(s_in, ev[0], 0));
    fail(cudaStreamWaitEvent(s_out, ev[0], 0));
    if (lengths) {
      fail(cudaMemcpyAsync(len_dev, lengths, static_cast<size_t>(batch) * 4, cudaMemcpyDefault,
                           s_in));
      for (int64_t ci = 0; memset32 && ci < nchunks; ++ci) {
        // the window's own length (read from the host array now): keys at or
        // past L_b stay masked in the window's coordinates
        const Chunk& c = p.chunks[ci];
        const int64_t L = std::min<int64_t>(std::max<int32_t>(lengths[c.b0], 0), n);
        const int64_t Lw = std::min<int64_t>(std::max<int64_t>(L - int64_t(c.a) * NB_BLOCK, 0),
                                             int64_t(c.w) * NB_BLOCK);
        if (memset32(reinterpret_cast<CUdeviceptr>(len_dev + batch + ci),
                     static_cast<unsigned int>(Lw), 1,
                     reinterpret_cast<CUstream>(s_in)) != CUDA_SUCCESS && st == NB_OK)
          st = NB_ERR_CUDA;
      }
    }
  }
  for (int64_t ci = 0; ci < nchunks && st == NB_OK; ++ci) {
    const Chunk& c = p.chunks[ci];
    const int64_t u0 = static_cast<int64_t>(c.b0) * heads + c.h0;  // first slice
    const int64_t units = static_cast<int64_t>(c.nbr) * c.nh;
    const int nw = c.w * NB_BLOCK;  // rows of each slice on the device
    uint8_t* slot = ws + p.len_bytes + static_cast<size_t>(ci % p.slots) * p.slot_bytes;
    uint8_t* dev[8];  // q k v dout o dq dk dv
    for (int i = 0; i < 8; ++i) dev[i] = slot + i * p.tensor;
    float* lse_dev = reinterpret_cast<float*>(slot + 8 * p.tensor);
    void* bws = slot + p.ws_off;
    const size_t bws_bytes = p.slot_bytes - p.ws_off;
    // host offsets of the copied rows (slices are contiguous; a window is one
    // slice's rows [a, a + w) in blocks)
    const int64_t in_row = u0 * n + static_cast<int64_t>(c.a) * NB_BLOCK;
    const int64_t in_rows = c.window ? nw : units * n;
    const int64_t out_row = u0 * n + static_cast<int64_t>(c.lo) * NB_BLOCK;
    const int64_t out_rows = c.window ? int64_t(c.hi - c.lo) * NB_BLOCK : units * n;
    const int64_t dev_out_row = c.window ? int64_t(c.lo - c.a) * NB_BLOCK : 0;
    // copy-in, once the slot's previous chunk has been copied out
    if (ci >= p.slots) fail(cudaStreamWaitEvent(s_in, ev_out(ci - p.slots), 0));
    const void* hin[4] = {q, k, v, dout};
    for (int i = 0; i < 4; ++i)
      fail(cudaMemcpyAsync(dev[i], static_cast<const uint8_t*>(hin[i]) + in_row * row,
                           in_rows * row, cudaMemcpyDefault, s_in));
    fail(cudaEventRecord(ev_in(ci), s_in));
    // compute on the caller's stream
    fail(cudaStreamWaitEvent(cs, ev_in(ci), 0));
    if (st != NB_OK) break;
    const int32_t* lens = !lengths ? nullptr : c.window ? len_dev + batch + ci : len_dev + c.b0;
    const int cb = c.nbr, ch = c.nh;
    nb_status r = causal ? nb_attn_fwd_causal(dev[0], dev[1], dev[2], dev[4], lse_dev, lens, cb, ch,
                                              nw, d, R, dtype, cs)
                         : nb_attn_fwd(dev[0], dev[1], dev[2], dev[4], lse_dev, lens, cb, ch, nw,
                                       d, R, dtype, cs);
    if (r == NB_OK)
      r = causal ? nb_attn_bwd_causal(dev[0], dev[1], dev[2], dev[4], dev[3], lse_dev, lens,
                                      dev[5], dev[6], dev[7], bws, bws_bytes, cb, ch, nw, d, R,
                                      dtype, cs)
                 : nb_attn_bwd(dev[0], dev[1], dev[2], dev[4], dev[3], lse_dev, lens, dev[5],
                               dev[6], dev[7], bws, bws_bytes, cb, ch, nw, d, R, dtype, cs);
    if (r != NB_OK) {
      st = r;
      break;
    }
    fail(cudaEventRecord(ev_comp(ci), cs));
    // copy-out of the owned rows
    fail(cudaStreamWaitEvent(s_out, ev_comp(ci), 0));
    void* hout[4] = {o, dq, dk, dv};
    const int src[4] = {4, 5, 6, 7};
    for (int i = 0; i < 4; ++i)
      fail(cudaMemcpyAsync(static_cast<uint8_t*>(hout[i]) + out_row * row,
                           dev[src[i]] + dev_out_row * row, out_rows * row, cudaMemcpyDefault,
                           s_out));
    if (lse)
      fail(cudaMemcpyAsync(lse + out_row, lse_dev + dev_out_row, out_rows * 4, cudaMemcpyDefault,
                           s_out));
    fail(cudaEventRecord(ev_out(ci), s_out));
  }
  // the caller's stream covers every copy-out (and, through them, every stage)
  if (st == NB_OK) {
    fail(cudaStreamWaitEvent(cs, ev_out(nchunks - 1), 0));
  } else {
    // an error after some work was queued: still order the caller's stream after
    // whatever was queued, so the workspace is not reused under it
    cudaEvent_t done_in = nullptr, done_out = nullptr;
    if (cudaEventCreateWithFlags(&done_in, cudaEventDisableTiming) == cudaSuccess &&
        cudaEventRecord(done_in, s_in) == cudaSuccess)
      cudaStreamWaitEvent(cs, done_in, 0);
    if (cudaEventCreateWithFlags(&done_out, cudaEventDisableTiming) == cudaSuccess &&
        cudaEventRecord(done_out, s_out) == cudaSuccess)
      cudaStreamWaitEvent(cs, done_out, 0);
    if (done_in) cudaEventDestroy(done_in);
    if (done_out) cudaEventDestroy(done_out);
  }
  // streams and events are released once their queued work completes
  for (auto& e : ev)
    if (e) cudaEventDestroy(e);
  cudaStreamDestroy(s_in);
  cudaStreamDestroy(s_out);
  return st;
}

}  // extern "C"
