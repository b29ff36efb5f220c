"""Benchmark of the hot path: k-mer tokenization of a batch plus banded
block-sparse local attention forward + backward, through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of every step of the path over one batch: nb_tokenize_kmer
on the batch's DNA (batch x (n + 5) bases), nb_attn_fwd and nb_attn_bwd.  The
headline workload is the largest single-GPU configuration, ``bf16_n1m``
(1 x 8 x 1048576 x 64, R = 8: the forward, then forward + backward).  Inputs
are seeded synthetic tensors resident in HBM; several input sets rotate so
that each step reads inputs that are not L2-resident.  Time is taken with
CUDA events on the launching stream, bracketed by a barrier and a device
synchronize, and the max over ranks is reported.  For N > 1 every rank
processes its own batch (weak scaling, no collective on the data path).

Rank 0 prints one JSON line.  At N = 1 the line also carries ``sub_results``:
the other configurations (fp32 1 x 1 x 256, the ragged-length bf16 batch,
the 131072-token d = 128 sequence and the 2**28-base tokenizer), each timed
the same way with its own roofline.  ``--impl reference`` times the CPU
oracle (fp64 NumPy) on a bounded sample of the same workload instead.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "block-sparse local attn fwd+bwd tokens/s and % of roofline (HBM or tensor)"
HEADLINE = "bf16_n1m"
SUB_WORKLOADS = ("fp32_n256", "bf16_varlen", "bf16_n131k", "dna_2p28")
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024
SUSTAINED_AFTER_S = 2.0  # a timed region at least this long is compared with the sustained peak
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "dram_traffic.json")


# ----------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(PEAKS_FALLBACK), "fallback"


def _strip_comments(src: str) -> str:
    """C/C++ source without comments and trailing blanks (traffic depends on the code only)."""
    import re

    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


# Host-only files that launch no kernel of their own and that no kernel file
# includes: changing them cannot change a kernel's DRAM traffic.
HOST_ONLY_SOURCES = ("attn_host.cu",)


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_local_nb_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name in HOST_ONLY_SOURCES:
            continue
        with open(os.path.join(csrc, name)) as f:
            h.update(name.encode() + _strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes (read + write) per launch of `kernel` on `workload`, from the
    JSON record of ncu captures, valid only while the kernel sources still hash
    to the value recorded with it (else None)."""
    try:
        with open(TRAFFIC_RECORD) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    src = kernel_source_hash()
    for r in rec.get("records", []):
        if r.get("kernel") == kernel and r.get("workload") == workload and r.get("source_hash") == src:
            try:
                return float(r["bytes_per_launch"])
            except (KeyError, TypeError, ValueError):
                return None
    return None


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.device_index = device_index
        self.lines = []

    def __enter__(self):
        try:
            import torch

            props = torch.cuda.get_device_properties(self.device_index)
            bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            sel = ["--id=" + bus]
        except Exception:
            sel = []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", *sel, "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- workload

def algorithmic(w, lengths):
    """Algorithmic bytes and flops of one call (valid rows and visible pairs only)."""
    e = 2 if w.dtype == "bf16" else 4
    nb_ = w.n // 32
    tok = 0
    pairs = 0
    for L in lengths:
        L = int(L)
        tok += L
        for i in range((L + 31) // 32):
            rows = min(32, L - 32 * i)
            lo = max(0, i - w.R)
            if getattr(w, "causal", False):  # row q sees keys lo*32 .. q
                pairs += sum(32 * i + r - lo * 32 + 1 for r in range(rows))
                continue
            hi = min(nb_ - 1, i + w.R)
            keys = min((hi + 1) * 32, L) - lo * 32
            pairs += rows * keys
    th = tok * w.heads
    pairs *= w.heads
    return {
        "tokens": tok,
        "fwd_bytes": th * (4 * w.d * e + 4),   # read Q K V, write O and lse
        "bwd_bytes": th * (8 * w.d * e + 8),   # read Q K V O dO, write dQ dK dV; row term D
        "fwd_flops": 4 * w.d * pairs,          # Q K^T and P V
        "bwd_flops": 10 * w.d * pairs,         # S, dP, dV, dK, dQ
        "pairs": pairs,
    }


def tokenizer_bytes(bases: int, k: int = 6) -> int:
    """Algorithmic bytes of nb_tokenize_kmer: 1 byte read per base, a uint16 ID
    written per window and the packed stream (one byte per four bases)."""
    return bases + 2 * max(bases - k + 1, 0) + (bases + 3) // 4


def dna_for_batch(w, seed):
    from block_sparse_local_nb_b200.inputs import make_dna

    return make_dna(w.batch * (w.n + 5), seed=seed)


def fp32_peak_tflops(sm_mhz):
    """CUDA-core fp32 FMA peak: SMs x 128 lanes x 2 flops x clock."""
    import torch

    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    return sms * 128 * 2 * (sm_mhz or 1965.0) * 1e6 / 1e12


def roofline(nbytes, flops, ms, peaks, timed_s, dtype, sm_max_mhz=None):
    """Fraction of the roofline of one call: the slower of its algorithmic
    bytes at HBM bandwidth and its algorithmic flops at the tensor (bf16) or
    fp32 FMA peak.  The bf16 peak is the burst figure for a timed region
    shorter than SUSTAINED_AFTER_S seconds, else the sustained figure."""
    hbm = float(peaks["hbm_gbs"])
    if dtype == "bf16":
        sustained = timed_s >= SUSTAINED_AFTER_S and "bf16_tflops_sustained" in peaks
        comp = float(peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"])
        comp_bound, comp_kind = "tensor", "sustained" if sustained else "burst"
    else:
        comp = fp32_peak_tflops(sm_max_mhz)
        comp_bound, comp_kind = "alu", "fp32 FMA: SMs x 128 x 2 x max SM clock"
    t_hbm = nbytes / (hbm * 1e9)
    t_comp = flops / (comp * 1e12)
    if t_hbm >= t_comp:
        achieved = nbytes / (ms / 1e3) / 1e9
        r = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s"}
    else:
        achieved = flops / (ms / 1e3) / 1e12
        r = {"bound": comp_bound, "achieved": achieved, "peak": comp, "unit": "TFLOP/s",
             "peak_kind": comp_kind}
    r["frac"] = r["achieved"] / r["peak"]
    r["roofline_ms"] = max(t_hbm, t_comp) * 1e3
    return r


# ------------------------------------------------------- oracle samples

def oracle_window(w, lengths, step):
    """(sequence, head, first block, end block) of the oracle sample of `step`:
    a whole sequence when it has at most 256 blocks, else a window of 256
    query blocks at a position that moves from step to step."""
    nb_ = w.n // 32
    b = step % w.batch
    h = (step // w.batch) % w.heads
    Lb = int(lengths[b])
    blocks = (Lb + 31) // 32
    if blocks <= 256:
        return b, h, 0, blocks
    lo = (step * 7919 * 32) % (blocks - 256 + 1)
    return b, h, lo, min(nb_, lo + 256)


def oracle_sample(w, fetch, lengths, dna, step):
    """Run the fp64 oracle (forward, backward, tokenization) on one sample and
    return the token-equivalents it covered (query rows of one head / heads).
    A window is evaluated with two band radii of context on each side, where
    the oracle's outputs for the window are exact.  ``fetch(b, h, r0, r1)``
    returns rows [r0, r1) of Q, K, V, dO of one head as fp64 [1, 1, rows, d]."""
    from oracle import attn_bwd_banded, attn_fwd_banded, kmer_ids, pack_2bit

    b, h, lo, hi = oracle_window(w, lengths, step)
    nb_ = w.n // 32
    s, e = max(0, lo - 2 * w.R), min(nb_, hi + 2 * w.R)
    Lb = int(lengths[b])
    Lsub = min(max(Lb - 32 * s, 0), 32 * (e - s))
    sub = fetch(b, h, 32 * s, 32 * e)
    attn_fwd_banded(*sub[:3], w.R, [Lsub], causal=w.causal)
    if w.backward:
        attn_bwd_banded(*sub, w.R, [Lsub], causal=w.causal)
    rows = max(0, min(Lb, 32 * hi) - 32 * lo)
    seg = dna[b * (w.n + 5) + 32 * lo: b * (w.n + 5) + 32 * lo + rows + 5]
    kmer_ids(seg, 6)
    pack_2bit(seg)
    return rows / w.heads


def window_fetcher(tensors):
    """fetch(b, h, r0, r1) over [batch, heads, n, d] tensors (CPU or device)."""
    def fetch(b, h, r0, r1):
        return [t[b:b + 1, h:h + 1, r0:r1].to("cpu", copy=True).double().numpy() for t in tensors]
    return fetch


def _blas_threads():
    from threadpoolctl import threadpool_info

    return max([p.get("num_threads", 1) for p in threadpool_info()] or [1])


def run_reference_arm(args, w):
    """Time the CPU oracle on a bounded sample of the workload (rank 0 only)."""
    from block_sparse_local_nb_b200.inputs import make_attn_inputs

    q, k, v, do, lengths = make_attn_inputs(w)
    fetch = window_fetcher((q, k, v, do))
    lengths = lengths.numpy()
    dna = dna_for_batch(w, seed=w.seed)
    for s in range(args.warmup):
        oracle_sample(w, fetch, lengths, dna, s)
    t0 = time.perf_counter()
    tok = 0.0
    for s in range(args.steps):
        tok += oracle_sample(w, fetch, lengths, dna, args.warmup + s)
    dt = time.perf_counter() - t0
    value = tok / dt
    cores = _blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": "per step: one head of one sequence (whole when at most 256 "
                                   "blocks, else a 256-block window of query blocks at a moving "
                                   "position, evaluated with 2R blocks of context on each side) "
                                   "through the fp64 banded oracle forward+backward plus the "
                                   "k-mer tokenization of its bases; counted as rows/heads tokens"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline(w, fetch, lengths, dna, budget_s=10.0):
    """Oracle timed on the host cores on a bounded sample (about `budget_s` of
    CPU work) of the benchmarked inputs."""
    t0 = time.perf_counter()
    tok = 0.0
    samples = 0
    while time.perf_counter() - t0 < budget_s:
        tok += oracle_sample(w, fetch, lengths, dna, samples)
        samples += 1
    dt = time.perf_counter() - t0
    return {"value": tok / dt, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{samples} samples in {dt:.1f} s, each one head of one sequence (whole when "
                      f"at most 256 blocks, else a 256-block window of query blocks with 2R "
                      f"blocks of context each side) through the fp64 banded oracle fwd+bwd plus "
                      f"the k-mer tokenization of its bases, counted as rows/heads tokens; host "
                      f"has {os.cpu_count()} logical cores"}


def check_kernel_error(nb):
    """A kernel that gave up on a bounded wait leaves a code in the library's
    error word; a timing that includes such a launch is not a measurement."""
    code = nb.nb_kernel_error(clear=True)
    if code:
        raise RuntimeError(f"a kernel recorded wait-timeout code {code:#x}: no valid timing")


def workload_config(w):
    return {"workload": w.name, "desc": w.desc + " + k=6 tokenization of the batch's "
            f"{w.batch}x({w.n}+5) bases", "batch": w.batch, "heads": w.heads, "n": w.n,
            "d": w.d, "R": w.R}


# ------------------------------------------------------------ GPU timing

def time_attention(w, args, dev, rank, world, with_e2e, steps, warmup):
    """Time `steps` steps (tokenize + fwd [+ bwd]) of workload `w` on `dev`;
    returns the measurements (max over ranks of the timed region)."""
    import torch
    import torch.distributed as dist

    import block_sparse_local_nb_b200 as nb
    from block_sparse_local_nb_b200.dist import job_throughput, max_over_ranks, rank_seed
    from block_sparse_local_nb_b200.inputs import make_attn_inputs

    dt_code = nb.NB_BF16 if w.dtype == "bf16" else nb.NB_F32
    B, H, N, D, R = w.batch, w.heads, w.n, w.d, w.R
    stream = torch.cuda.Stream(device=dev)
    base_seed = rank_seed(w.seed, rank)
    q0, k0, v0, do0, lengths = make_attn_inputs(w, device=dev, seed=base_seed)
    lengths_d = lengths.to(dev)
    dna_np = dna_for_batch(w, seed=base_seed)
    elem = q0.element_size()
    ws_bytes = nb.attn_bwd_workspace_size(B, H, N, D, dt_code) if w.backward else 0
    set_bytes = 8 * q0.numel() * elem + 2 * B * H * N * 4 + ws_bytes + 3 * dna_np.size
    nsets = args.sets if args.sets > 0 else max(1, min(8, math.ceil(3 * L2_BYTES / set_bytes) + 1))
    sets = []
    for s in range(nsets):
        if s == 0:
            q, k, v, do = q0, k0, v0, do0
        else:
            q, k, v, do, _ = make_attn_inputs(w, device=dev, seed=base_seed + s)
        st = {"q": q, "k": k, "v": v, "do": do, "o": torch.empty_like(q),
              "lse": torch.empty((B, H, N), dtype=torch.float32, device=dev),
              "dna": torch.from_numpy(dna_np).to(dev),
              "ids": torch.empty(dna_np.size - 5, dtype=torch.int16, device=dev),
              "packed": torch.empty((dna_np.size + 3) // 4, dtype=torch.uint8, device=dev)}
        if w.backward:
            st.update(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
                      ws=torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev))
        sets.append(st)
    torch.cuda.synchronize(dev)

    sptr = stream.cuda_stream
    fwd = nb.nb_attn_fwd_causal if w.causal else nb.nb_attn_fwd
    bwd = nb.nb_attn_bwd_causal if w.causal else nb.nb_attn_bwd

    def step(st, ev=None):
        if ev is not None:
            ev[0].record(stream)
        nb.nb_tokenize_kmer(st["dna"], st["dna"].numel(), st["ids"], st["packed"], 6, sptr)
        if ev is not None:
            ev[1].record(stream)
        fwd(st["q"], st["k"], st["v"], st["o"], st["lse"], lengths_d, B, H, N, D, R, dt_code, sptr)
        if ev is not None:
            ev[2].record(stream)
        if w.backward:
            bwd(st["q"], st["k"], st["v"], st["o"], st["do"], st["lse"], lengths_d, st["dq"],
                st["dk"], st["dv"], st["ws"], ws_bytes, B, H, N, D, R, dt_code, sptr)
        if ev is not None:
            ev[3].record(stream)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[dev.index])
        torch.cuda.synchronize(dev)

    with torch.cuda.stream(stream):
        for s in range(warmup):
            step(sets[s % nsets])
    barrier()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index)
    with sampler:
        barrier()
        start.record(stream)
        for s in range(steps):
            step(sets[s % nsets], evs[s])
        end.record(stream)
        barrier()
    elapsed_ms = max_over_ranks(start.elapsed_time(end), dev)
    check_kernel_error(nb)
    alg = algorithmic(w, lengths.tolist())
    res = {
        "w": w, "alg": alg, "elapsed_ms": elapsed_ms, "steps": steps, "nsets": nsets,
        "set_bytes": set_bytes, "dna_bases": int(dna_np.size),
        "value": job_throughput(alg["tokens"], steps, world, elapsed_ms),
        "calls_ms": {
            "nb_tokenize_kmer": statistics.mean(e[0].elapsed_time(e[1]) for e in evs),
            "nb_attn_fwd": statistics.mean(e[1].elapsed_time(e[2]) for e in evs),
            "nb_attn_bwd": statistics.mean(e[2].elapsed_time(e[3]) for e in evs) if w.backward else 0.0,
        },
        "clocks": sampler.summary(),
        "launches_per_step": 2 + (3 if w.backward else 0),
    }
    res["inputs"] = (sets[0]["q"], sets[0]["k"], sets[0]["v"], sets[0]["do"])
    res["lengths"] = lengths.numpy()
    res["dna"] = dna_np
    if not with_e2e:
        del sets
        return res

    # ---- end to end through the C ABI with host buffers (pinned), copies timed.
    # Attention with a backward goes through nb_attn_fwd_bwd_host, which takes
    # the host tensors and overlaps their copies with the kernels chunk by
    # chunk; the tokenizer's bases and outputs (and a forward-only workload's
    # tensors) are copied with plain asynchronous copies around the device calls.
    st = sets[0]
    for extra in sets[1:]:
        extra.clear()
    torch.cuda.empty_cache()
    host = {name: st[name].cpu().pin_memory() for name in ("q", "k", "v", "do")}
    host["dna"] = torch.from_numpy(dna_np).pin_memory()
    host["lengths"] = lengths.to(torch.int32).pin_memory()
    out_names = ("o", "lse", "ids", "packed") + (("dq", "dk", "dv") if w.backward else ())
    outs = {name: torch.empty_like(st[name], device="cpu").pin_memory() for name in out_names}
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in outs.values())
    if w.backward:
        for name in ("q", "k", "v", "do", "o", "lse", "dq", "dk", "dv", "ws"):
            st.pop(name)
        torch.cuda.empty_cache()
        hws_bytes = nb.attn_fwd_bwd_host_workspace_size(B, H, N, D, R, dt_code)
        hws = torch.empty(hws_bytes, dtype=torch.uint8, device=dev)
    e_steps = max(1, min(steps, 5))
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        def e2e_step():
            st["dna"].copy_(host["dna"], non_blocking=True)
            nb.nb_tokenize_kmer(st["dna"], st["dna"].numel(), st["ids"], st["packed"], 6, sptr)
            for name in ("ids", "packed"):
                outs[name].copy_(st[name], non_blocking=True)
            if w.backward:
                nb.nb_attn_fwd_bwd_host(host["q"], host["k"], host["v"], host["do"],
                                        host["lengths"], outs["o"], outs["lse"], outs["dq"],
                                        outs["dk"], outs["dv"], hws, hws_bytes, B, H, N, D, R,
                                        dt_code, w.causal, sptr)
            else:
                for name in ("q", "k", "v"):
                    st[name].copy_(host[name], non_blocking=True)
                lengths_d.copy_(host["lengths"], non_blocking=True)
                fwd(st["q"], st["k"], st["v"], st["o"], st["lse"], lengths_d, B, H, N, D, R,
                    dt_code, sptr)
                for name in ("o", "lse"):
                    outs[name].copy_(st[name], non_blocking=True)
        for _ in range(2):
            e2e_step()
        barrier()
        e_start.record(stream)
        for _ in range(e_steps):
            e2e_step()
        e_end.record(stream)
        barrier()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end), dev)
    check_kernel_error(nb)
    res["e2e"] = {"value": job_throughput(alg["tokens"], e_steps, world, e2e_ms), "unit": "tokens/s",
                  "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e_steps,
                  "path": ("nb_attn_fwd_bwd_host on pinned host tensors (chunked copy-in / compute / "
                           "copy-out overlap) + nb_tokenize_kmer with plain copies" if w.backward else
                           "plain copies around nb_tokenize_kmer and nb_attn_fwd")}
    del sets, host, outs
    return res


def time_host_link(nbytes=1 << 30, reps=5):
    """Host link bandwidth with pinned buffers: host->device alone, device->host
    alone, and both at once on two streams (GB/s per direction, CUDA events)."""
    import torch

    h_src = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    h_dst = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    d_a = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    d_b = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def run(h2d, d2h):
        main = torch.cuda.current_stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for timed in (False, True):
            torch.cuda.synchronize()
            e0.record(main)
            s_in.wait_stream(main)
            s_out.wait_stream(main)
            for _ in range(reps if timed else 2):
                if h2d:
                    with torch.cuda.stream(s_in):
                        d_a.copy_(h_src, non_blocking=True)
                if d2h:
                    with torch.cuda.stream(s_out):
                        h_dst.copy_(d_b, non_blocking=True)
            main.wait_stream(s_in)
            main.wait_stream(s_out)
            e1.record(main)
        torch.cuda.synchronize()
        return nbytes * reps / (e0.elapsed_time(e1) * 1e-3) / 1e9

    return {"metric": "host link bandwidth, pinned cudaMemcpyAsync", "unit": "GB/s per direction",
            "bytes_per_copy": nbytes, "h2d": run(True, False), "d2h": run(False, True),
            "both_at_once": run(True, True)}


def attention_line(res, peaks, peak_kind, world):
    """The JSON fields of one attention workload's measurement."""
    w, alg = res["w"], res["alg"]
    steps = res["steps"]
    ms_step = res["elapsed_ms"] / steps
    timed_s = res["elapsed_ms"] / 1e3
    smax = res["clocks"].get("sm_max_mhz")
    calls = {}
    fwd_ms, bwd_ms, tok_ms = (res["calls_ms"][c] for c in ("nb_attn_fwd", "nb_attn_bwd", "nb_tokenize_kmer"))
    calls["nb_attn_fwd"] = roofline(alg["fwd_bytes"], alg["fwd_flops"], fwd_ms, peaks, timed_s, w.dtype, smax)
    if w.backward:
        calls["nb_attn_bwd"] = roofline(alg["bwd_bytes"], alg["bwd_flops"], bwd_ms, peaks, timed_s,
                                        w.dtype, smax)
    calls["nb_tokenize_kmer"] = roofline(tokenizer_bytes(res["dna_bases"]), 0, tok_ms, peaks,
                                         timed_s, "u8")
    for name, ms in res["calls_ms"].items():
        if name in calls:
            calls[name]["ms"] = ms
    dom = "nb_attn_bwd" if w.backward and bwd_ms >= fwd_ms else "nb_attn_fwd"
    roof = dict(calls[dom])
    roof.pop("ms", None)
    roof["traffic"] = recorded_traffic(dom, w.name)
    roof["kernel"] = dom
    roof["peak_source"] = f"{peak_kind} ({'MEASURED_PEAKS.json' if peak_kind == 'measured' else 'fallback'})"
    step_bytes = alg["fwd_bytes"] + (alg["bwd_bytes"] if w.backward else 0) + tokenizer_bytes(res["dna_bases"])
    step_flops = alg["fwd_flops"] + (alg["bwd_flops"] if w.backward else 0)
    step_roof = roofline(step_bytes, step_flops, ms_step, peaks, timed_s, w.dtype, smax)
    cfg = workload_config(w)
    cfg.update({"tokens_per_step": alg["tokens"],
                "parallelism": f"dp{world} (independent batches)",
                "l2": f"{res['nsets']} rotating input sets of {res['set_bytes'] / 2**20:.0f} MiB each "
                      f"(> {L2_BYTES >> 20} MiB L2 between reuses)"})
    return {
        "value": res["value"], "unit": "tokens/s", "ms_per_step": ms_step,
        "dtype": w.dtype, "config": cfg, "roofline": roof,
        "step_roofline": {"bytes": step_bytes, "flops": step_flops, "bound": step_roof["bound"],
                          "frac": step_roof["frac"], "roofline_ms": step_roof["roofline_ms"]},
        "calls": calls, "clocks": res["clocks"],
        "gpu_launches": res["launches_per_step"] * steps,
    }


def time_tokenizer(args, dev, steps, warmup):
    """The 2**28-byte k-mer tokenizer workload alone: bases/s and the fraction
    of the HBM roofline (1 byte read + 2.25 bytes written per base)."""
    import torch

    import block_sparse_local_nb_b200 as nb
    from block_sparse_local_nb_b200.inputs import DNA_BYTES, make_dna

    dna = make_dna(DNA_BYTES)
    seq = torch.from_numpy(dna).to(dev)
    ids = torch.empty(DNA_BYTES - 5, dtype=torch.int16, device=dev)
    packed = torch.empty(DNA_BYTES // 4, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    sptr = stream.cuda_stream
    for _ in range(warmup):
        nb.nb_tokenize_kmer(seq, DNA_BYTES, ids, packed, 6, sptr)
    torch.cuda.synchronize(dev)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index)
    with sampler:
        start.record(stream)
        for _ in range(steps):
            nb.nb_tokenize_kmer(seq, DNA_BYTES, ids, packed, 6, sptr)
        end.record(stream)
        torch.cuda.synchronize(dev)
    check_kernel_error(nb)
    ms = start.elapsed_time(end) / steps
    peaks, peak_kind = load_peaks()
    roof = roofline(tokenizer_bytes(DNA_BYTES), 0, ms, peaks, ms * steps / 1e3, "u8")
    roof.update(traffic=recorded_traffic("tokenize_kmer_kernel", "dna_2p28"),
                kernel="tokenize_kmer_kernel", peak_source=peak_kind)
    out = {
        "metric": "k-mer tokenizer bases/s and % of HBM roofline", "value": DNA_BYTES / (ms / 1e3),
        "unit": "bases/s", "ms_per_step": ms, "steps": steps, "dtype": "u8",
        "config": {"workload": "dna_2p28", "bytes": DNA_BYTES, "k": 6, "n_fraction": 0.01,
                   "l2": "inputs and outputs (872 MB) larger than the 126 MB L2"},
        "roofline": roof, "gpu_launches": steps, "clocks": sampler.summary(),
    }
    del seq, ids, packed
    torch.cuda.empty_cache()
    if not args.no_cpu_baseline:
        from oracle import kmer_ids, pack_2bit

        sample = dna[: 1 << 24]
        t0 = time.perf_counter()
        kmer_ids(sample, 6)
        pack_2bit(sample)
        dt = time.perf_counter() - t0
        out["cpu_baseline"] = {"value": sample.size / dt, "unit": "bases/s", "cores": 1,
                               "kind": "oracle", "sample": "first 2**24 bytes of the workload "
                               "through the NumPy oracle (ids + packed stream)"}
    return out


def run_batch_ids_workload(args):
    """The batch-to-model-IDs tokenizer alone (one GPU): windows/s and the
    fraction of the HBM roofline (bases and offsets read, padded int64 IDs and
    lengths written)."""
    import numpy as np
    import torch

    import block_sparse_local_nb_b200 as nb
    from block_sparse_local_nb_b200.inputs import make_dna_batch

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    blob, offsets = make_dna_batch()
    batch = offsets.size - 1
    windows = np.maximum(np.diff(offsets) - 5, 0)
    n_pad = nb.nb_batch_ceiling(offsets, batch, 6)
    seqs = torch.from_numpy(blob).to(dev)
    off = torch.from_numpy(offsets).to(dev)
    ids = torch.empty((batch, n_pad), dtype=torch.int64, device=dev)
    lengths = torch.empty(batch, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    sptr = stream.cuda_stream
    for _ in range(args.warmup):
        nb.nb_tokenize_batch(seqs, off, batch, 6, ids, lengths, n_pad, sptr)
    torch.cuda.synchronize(dev)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(0)
    with sampler:
        start.record(stream)
        for _ in range(args.steps):
            nb.nb_tokenize_batch(seqs, off, batch, 6, ids, lengths, n_pad, sptr)
        end.record(stream)
        torch.cuda.synchronize(dev)
    ms = start.elapsed_time(end) / args.steps
    peaks, peak_kind = load_peaks()
    alg_bytes = blob.size + 8 * offsets.size + 8 * batch * n_pad + 4 * batch
    roof = roofline(alg_bytes, 0, ms, peaks, ms * args.steps / 1e3, "u8")
    roof.update(traffic=recorded_traffic("tokenize_batch_kernel", "dna_batch_ids"),
                kernel="tokenize_batch_kernel", peak_source=peak_kind)
    line = {
        "metric": "batch tokenizer to model IDs windows/s and % of HBM roofline",
        "value": float(windows.sum()) / (ms / 1e3), "unit": "windows/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int64", "data": "synthetic",
        "config": {"workload": "dna_batch_ids", "sequences": int(batch), "bases": int(blob.size),
                   "n_pad": n_pad, "k": 6, "n_fraction": 0.01,
                   "l2": f"output ({8 * batch * n_pad / 2**20:.0f} MiB) larger than the 126 MB L2"},
        "roofline": roof, "gpu_launches": args.steps, "clocks": sampler.summary(),
    }
    if not args.no_cpu_baseline:
        from oracle.tokenizer import model_ids_batch

        sample = [blob[offsets[i]:offsets[i + 1]].tobytes() for i in range(256)]
        t0 = time.perf_counter()
        model_ids_batch(sample, 6, n_pad=n_pad)
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": float(windows[:256].sum()) / dt, "unit": "windows/s",
                                "cores": 1, "kind": "oracle",
                                "sample": "first 256 sequences through the NumPy oracle"}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--sets", type=int, default=0, help="rotating input sets (0 = auto)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub", action="store_true", help="headline workload only")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end (host buffers) measurement, for quick comparisons")
    ap.add_argument("--link", action="store_true",
                    help="only measure the host link: pinned copies host->device, "
                         "device->host and both at once (the end-to-end ceiling)")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="override n of a full-length workload (a smaller case of the same "
                         "shape, e.g. for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    from block_sparse_local_nb_b200.inputs import WORKLOADS

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.link:
        if rank == 0:
            print(json.dumps(time_host_link()), flush=True)
        return
    if args.workload == "dna_batch_ids":
        if args.impl == "native" and rank == 0:
            run_batch_ids_workload(args)
        return
    if args.workload == "dna_2p28":
        if args.impl == "native" and rank == 0:
            import torch

            dev = torch.device("cuda", 0)
            torch.cuda.set_device(dev)
            line = time_tokenizer(args, dev, args.steps, args.warmup)
            line.update(n_gpus=1, warmup=args.warmup, higher_is_better=True, scaling="weak",
                        vs_baseline=None, data="synthetic")
            print(json.dumps(line), flush=True)
        return
    w = WORKLOADS[args.workload]
    if args.seq_len:
        if w.varlen is not None or args.seq_len % 32:
            ap.error("--seq-len applies to full-length workloads and must be a multiple of 32")
        import dataclasses

        w = dataclasses.replace(w, n=args.seq_len, name=f"{w.name}@n{args.seq_len}",
                                desc=w.desc.replace(str(w.n), str(args.seq_len)))

    if args.impl == "reference":
        if rank == 0:
            run_reference_arm(args, w)
        return

    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    res = time_attention(w, args, dev, rank, world, not args.no_e2e, args.steps, args.warmup)
    if world > 1:
        dist.barrier(device_ids=[local_rank])
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_kind = load_peaks()
    body = attention_line(res, peaks, peak_kind, world)
    line = {
        "metric": METRIC, "value": body["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": body["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic", "config": body["config"], "roofline": body["roofline"],
        "step_roofline": body["step_roofline"], "calls": body["calls"], "e2e": res.get("e2e"),
        "gpu_launches": body["gpu_launches"], "clocks": body["clocks"],
    }
    if world == 1 and not args.no_sub:
        subs = {}
        for name in SUB_WORKLOADS:
            if name == args.workload:
                continue
            if name == "dna_2p28":
                subs[name] = time_tokenizer(args, dev, max(args.steps, 20), args.warmup)
                continue
            sw = WORKLOADS[name]
            sres = time_attention(sw, args, dev, 0, 1, False, max(args.steps, 20), args.warmup)
            sres.pop("inputs")
            torch.cuda.empty_cache()
            sub = attention_line(sres, peaks, peak_kind, 1)
            sub["metric"] = METRIC
            subs[name] = sub
        line["sub_results"] = subs
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, window_fetcher(res["inputs"]), res["lengths"],
                                            res["dna"])
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
