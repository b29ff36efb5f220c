// Forward + backward on host-resident tensors (nb_attn_fwd_bwd_host): the
// problem is cut into chunks of whole (batch, head) slices, which attention
// treats independently, and every chunk goes through three stages on three
// streams: copy-in (q, k, v, dO), compute (nb_attn_fwd then nb_attn_bwd on the
// caller's stream) and copy-out (O, lse, dQ, dK, dV).  Chunk i + 1 is copied
// in while chunk i computes and chunk i - 1 is copied out, so the host link
// carries both directions at once and the kernels hide behind the copies.
// The device side holds NSLOT chunks at a time in the caller's workspace.
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "../../include/nb.h"
#include "nb_internal.h"

namespace {

constexpr int kSlots = 3;        // chunks resident on the device at once
constexpr int64_t kChunks = 8;   // aim: this many chunks (pipeline depth)

struct Plan {
  int64_t units;      // batch * heads slices of n x d
  int rows_per;       // > 0: a chunk is rows_per whole batch rows
  int heads_per;      // > 0: a chunk is heads_per heads of one batch row
  int64_t max_units;  // slices in the largest chunk
  int64_t nchunks;
  int slots;
  size_t len_bytes;   // device copy of lengths
  size_t slot_bytes;  // one chunk's tensors + backward workspace
  size_t ws_off;      // offset of the backward workspace inside a slot
};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

Plan make_plan(int batch, int heads, int n, int d) {
  Plan p{};
  p.units = static_cast<int64_t>(batch) * heads;
  const int64_t target = (p.units + kChunks - 1) / kChunks;
  if (target >= heads) {
    p.rows_per = static_cast<int>(target / heads);
    p.max_units = static_cast<int64_t>(p.rows_per) * heads;
    p.nchunks = (batch + p.rows_per - 1) / p.rows_per;
  } else {
    p.heads_per = static_cast<int>(target);
    p.max_units = p.heads_per;
    p.nchunks = static_cast<int64_t>(batch) * ((heads + p.heads_per - 1) / p.heads_per);
  }
  p.slots = static_cast<int>(p.nchunks < kSlots ? p.nchunks : kSlots);
  p.len_bytes = up256(static_cast<size_t>(batch) * 4);
  const size_t tensor = up256(static_cast<size_t>(p.max_units) * n * d * 2);
  const size_t lse = up256(static_cast<size_t>(p.max_units) * n * 4);
  p.ws_off = 8 * tensor + lse;
  p.slot_bytes = p.ws_off + up256(nb::bwd_workspace_bytes(p.max_units * n, d));
  return p;
}

// Chunk c as (first batch row, rows, first head, heads).
void chunk_shape(const Plan& p, int heads, int64_t c, int& b0, int& nb_, int& h0, int& nh) {
  if (p.rows_per > 0) {
    b0 = static_cast<int>(c * p.rows_per);
    nb_ = p.rows_per;
    h0 = 0;
    nh = heads;
  } else {
    const int per_row = (heads + p.heads_per - 1) / p.heads_per;
    b0 = static_cast<int>(c / per_row);
    nb_ = 1;
    h0 = static_cast<int>(c % per_row) * p.heads_per;
    nh = p.heads_per;
    if (h0 + nh > heads) nh = heads - h0;
  }
}

bool shape_ok(int batch, int heads, int n, int d, int dtype) {
  // the same shape rules as nb_attn_bwd (which the compute stage calls)
  return nb_attn_bwd_workspace_size(batch, heads, n, d, dtype) > 0 && dtype == NB_BF16;
}

}  // namespace

extern "C" {

size_t nb_attn_fwd_bwd_host_workspace_size(int batch, int heads, int n, int d, int dtype) {
  if (!shape_ok(batch, heads, n, d, dtype)) return 0;
  const Plan p = make_plan(batch, heads, n, d);
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
      workspace_bytes < nb_attn_fwd_bwd_host_workspace_size(batch, heads, n, d, dtype))
    return NB_ERR_WORKSPACE;
  const nb_status dev_st = nb::device_check();
  if (dev_st != NB_OK) return dev_st;

  const Plan p = make_plan(batch, heads, n, d);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* len_dev = lengths ? reinterpret_cast<int32_t*>(ws) : nullptr;
  const size_t slice = static_cast<size_t>(n) * d * 2;  // bytes of one (b, h) slice
  const size_t tensor = up256(static_cast<size_t>(p.max_units) * slice);

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
  ev.resize(1 + 3 * p.nchunks, nullptr);
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
    if (len_dev)
      fail(cudaMemcpyAsync(len_dev, lengths, static_cast<size_t>(batch) * 4, cudaMemcpyDefault,
                           s_in));
  }
  for (int64_t c = 0; c < p.nchunks && st == NB_OK; ++c) {
    int b0, nbr, h0, nh;
    chunk_shape(p, heads, c, b0, nbr, h0, nh);
    if (b0 + nbr > batch) nbr = batch - b0;
    const int64_t u0 = static_cast<int64_t>(b0) * heads + h0;  // first slice
    const int64_t units = static_cast<int64_t>(nbr) * nh;
    const size_t bytes = static_cast<size_t>(units) * slice;
    uint8_t* slot = ws + p.len_bytes + static_cast<size_t>(c % p.slots) * p.slot_bytes;
    uint8_t* dev[8];  // q k v dout o dq dk dv
    for (int i = 0; i < 8; ++i) dev[i] = slot + i * tensor;
    float* lse_dev = reinterpret_cast<float*>(slot + 8 * tensor);
    void* bws = slot + p.ws_off;
    const size_t bws_bytes = p.slot_bytes - p.ws_off;
    const size_t off = static_cast<size_t>(u0) * slice;
    // copy-in, once the slot's previous chunk has been copied out
    if (c >= p.slots) fail(cudaStreamWaitEvent(s_in, ev_out(c - p.slots), 0));
    const void* hin[4] = {q, k, v, dout};
    for (int i = 0; i < 4; ++i)
      fail(cudaMemcpyAsync(dev[i], static_cast<const uint8_t*>(hin[i]) + off, bytes,
                           cudaMemcpyDefault, s_in));
    fail(cudaEventRecord(ev_in(c), s_in));
    // compute on the caller's stream
    fail(cudaStreamWaitEvent(cs, ev_in(c), 0));
    if (st != NB_OK) break;
    const int32_t* lens = len_dev ? len_dev + b0 : nullptr;
    const int cb = nbr, ch = nh;
    nb_status r = causal ? nb_attn_fwd_causal(dev[0], dev[1], dev[2], dev[4], lse_dev, lens, cb, ch,
                                              n, d, R, dtype, cs)
                         : nb_attn_fwd(dev[0], dev[1], dev[2], dev[4], lse_dev, lens, cb, ch, n,
                                       d, R, dtype, cs);
    if (r == NB_OK)
      r = causal ? nb_attn_bwd_causal(dev[0], dev[1], dev[2], dev[4], dev[3], lse_dev, lens,
                                      dev[5], dev[6], dev[7], bws, bws_bytes, cb, ch, n, d, R,
                                      dtype, cs)
                 : nb_attn_bwd(dev[0], dev[1], dev[2], dev[4], dev[3], lse_dev, lens, dev[5],
                               dev[6], dev[7], bws, bws_bytes, cb, ch, n, d, R, dtype, cs);
    if (r != NB_OK) {
      st = r;
      break;
    }
    fail(cudaEventRecord(ev_comp(c), cs));
    // copy-out
    fail(cudaStreamWaitEvent(s_out, ev_comp(c), 0));
    void* hout[4] = {o, dq, dk, dv};
    const int src[4] = {4, 5, 6, 7};
    for (int i = 0; i < 4; ++i)
      fail(cudaMemcpyAsync(static_cast<uint8_t*>(hout[i]) + off, dev[src[i]], bytes,
                           cudaMemcpyDefault, s_out));
    if (lse)
      fail(cudaMemcpyAsync(lse + u0 * n, lse_dev, static_cast<size_t>(units) * n * 4,
                           cudaMemcpyDefault, s_out));
    fail(cudaEventRecord(ev_out(c), s_out));
  }
  // the caller's stream covers every copy-out (and, through them, every stage)
  if (st == NB_OK) {
    fail(cudaStreamWaitEvent(cs, ev_out(p.nchunks - 1), 0));
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
