"""Benchmark of the HySparse hybrid block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload moe64k]
                    [--impl ours|reference] [--no-cpu-baseline] [--no-decode]
                    [--profile-stage full|topk|sparse]

One step = one hybrid block over one batch of synthetic input: the full
causal GQA layer with importance scores (row chunks), per-row top-k, then
N sparse layers (global top-k branch + 128-token window + gate), each stage
through the library's C ABI.  Prints ONE JSON line on rank 0.  The default
workload is the largest single-GPU configuration (moe64k: 65536-token
prefill, 64 query / 4 KV heads, 9 sparse layers); a prefill line also carries
the decode step (64 sequences x 32768-token caches) under "decode".

Multi-GPU: one process per GPU (torchrun).  Blocks are independent problems,
so every rank runs its own replica of the workload with no collective on the
data path ("scaling": "weak"); the timed region is bracketed by a barrier and
device synchronisation and the slowest rank's time is reported.

``--impl reference`` times the CPU oracle (there is no other implementation
of this method to run) on a bounded sample of query rows of the same
workload, extrapolated to the whole workload with the exact per-row cost.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "hybrid-block tokens/s (prefill) & decode step us; TFLOPS / HBM GB/s vs peak"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (the slowest rank's time).
    Uses the process group's backend: NCCL with a CUDA tensor, gloo on CPU."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class ClockSampler:
    """Samples SM clock and throttle reasons of one GPU through NVML while
    the timed region runs (reading only; no setting is changed)."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            try:
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId_v2(bus.encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report without clocks
            self.err = str(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.reasons |= int(r)
            except Exception:
                pass
            time.sleep(0.05)

    def __enter__(self):
        if self.ok:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for n, bit in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def code_only(text: str) -> str:
    """Source text without comments and blank lines, so that a recorded
    measurement of a kernel survives edits to its comments."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (ln.split("//", 1)[0].rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln.strip())


def source_hash(*names):
    """sha1 (12 hex digits) of the named kernel sources' code, comments and
    blank lines left out."""
    h = hashlib.sha1()
    for n in names:
        p = os.path.join(ROOT, "hybrid_sparse_attention_tcgen05_b200", "csrc", n)
        if os.path.exists(p):
            h.update(code_only(open(p, encoding="utf-8").read()).encode())
    return h.hexdigest()[:12]


def read_traffic(kernel_key: str, src_hash: str):
    """DRAM bytes per launch recorded from an ncu capture in
    profiles/traffic.txt ("<workload>/<kernel> <source-hash> <bytes-per-launch>");
    None if absent, taken on another workload size or taken on another version
    of the kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    for line in open(p):
        parts = line.split()
        if len(parts) >= 3 and parts[0] == kernel_key and parts[1] == src_hash:
            return float(parts[2])
    return None


def measure_l2(dev, mb: int = 64, passes: int = 8, reps: int = 5):
    """L2 read bandwidth on this GPU, measured live: the library's probe over
    an L2-resident buffer of `mb` MiB -- streaming 16-byte reads and random
    whole 256-byte rows, each through registers (ld.global.cg, 4 CTAs of 512
    threads per SM) and through cp.async into shared memory (one CTA of 7
    warps per SM, as the row-gather kernel reads) -- best of `reps` timed calls
    after one untimed call that makes the buffer resident.  The peak is the
    best of the four."""
    import hybrid_sparse_attention_tcgen05_b200 as hs
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    buf = torch.ones(mb << 20, dtype=torch.uint8, device=dev)
    sink = torch.zeros(4 * sms, dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream(dev)
    out = {"buffer_mib": mb, "passes_per_call": passes}
    for mode, key in ((0, "stream_gbs"), (1, "row_gather_gbs"), (2, "cp_async_stream_gbs"),
                      (3, "cp_async_row_gather_gbs")):
        blocks = 4 * sms if mode < 2 else sms
        hs.probe_l2_read(buf, 1, mode, blocks, sink)
        best = 0.0
        for _ in range(reps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            hs.probe_l2_read(buf, passes, mode, blocks, sink)
            e1.record(stream)
            torch.cuda.synchronize()
            best = max(best, passes * buf.numel() / (e0.elapsed_time(e1) / 1e3) / 1e9)
        out[key] = best
    out["peak_gbs"] = max(out[k] for k in ("stream_gbs", "row_gather_gbs", "cp_async_stream_gbs",
                                             "cp_async_row_gather_gbs"))
    del buf, sink
    return out


# ------------------------------------------------------------- work model

def pairs_causal(w):
    """Number of causal (row, key) pairs per (batch, head)."""
    tot = 0
    off = w.Lkv - w.Lq
    # sum_{i} (off + i + 1)
    tot = w.Lq * (off + 1) + w.Lq * (w.Lq - 1) // 2
    return tot


def sum_min(w, cap):
    """sum over rows of min(cap, pos+1)."""
    off = w.Lkv - w.Lq
    s = 0
    # rows with pos+1 <= cap: pos+1 = off+i+1 <= cap -> i <= cap-off-1
    n_small = max(0, min(w.Lq, cap - off))
    if n_small > 0:
        s += n_small * (off + 1) + n_small * (n_small - 1) // 2
    s += (w.Lq - n_small) * cap
    return s


def work_model(w):
    """Algorithmic work per step (what the method must do)."""
    P = pairs_causal(w)
    esz = 2 if w.dtype == "bf16" else 4
    flops_full = 4.0 * w.d * w.Hq * P * w.B                  # QK^T + PV
    flops_score = 2.0 * w.d * w.Hq * P * w.B                 # QK^T again
    score_bytes = 4.0 * P * w.Hkv * w.B * 2                  # written once, read once
    keff = sum_min(w, w.topk)
    weff = sum_min(w, w.window)
    gather = float(keff + weff) * w.Hkv * w.B * 2 * w.d * esz   # K and V rows per (row, kv head)
    io_sparse = float(w.B * w.Lq * w.Hq * w.d * esz * 2 + w.B * w.Lq * w.Hq * 4)
    idx_bytes = 4.0 * w.B * w.Hkv * w.Lq * w.topk
    kv_bytes = 2.0 * w.B * w.Lkv * w.Hkv * w.d * esz
    return {"flops_full_scores": flops_full + flops_score, "flops_full_fwd": flops_full,
            "score_bytes": score_bytes, "gather_bytes_per_layer": gather + io_sparse + idx_bytes,
            "kv_bytes": kv_bytes, "keff": keff, "weff": weff, "pairs": P}


# kernel sources of the gather sparse layer (their hash keys the traffic record)
SPARSE_GATHER_SRCS = ("sparse_mma.cu", "tc_util.cuh")


def l2_served(w):
    """The gather reads one KV head's K and V at a time; when that slice
    (B*Lkv*d*2 bytes each) fits comfortably in L2 its rows are L2 hits."""
    esz = 2 if w.dtype == "bf16" else 4
    return w.Lq > 1 and 2 * w.B * w.Lkv * w.d * esz <= 64 * 2 ** 20


def e2e_step_count(ms_per_step):
    """Steps of the end-to-end loop: about 6 s of device time, 4 to 64 steps,
    so that the copy pipeline's fill and drain are a small share of it
    (ms_per_step is the max over ranks, so every rank runs the same count)."""
    return int(max(4, min(64, 6000.0 / max(ms_per_step, 1e-3))))


def causal_tiles(Lq, Lkv, block=128):
    """128 x 128 tiles of the Lq x Lkv score matrix that hold at least one
    causal pair (row i sees keys 0 .. Lkv - Lq + i): the tiles a dense causal
    pass runs, the count behind the dense-or-gather estimate and the executed
    FLOPs of the dense-masked sparse layer."""
    off = Lkv - Lq
    return sum((off + min(Lq, block * (t + 1)) - 1) // block + 1 for t in range((Lq + block - 1) // block))


def sparse_path_is_dense(w):
    """The library's choice between the dense-masked and the gather sparse
    kernel (same estimate as hysparse_api.cu; HYSPARSE_SPARSE_PATH overrides)."""
    env = os.environ.get("HYSPARSE_SPARSE_PATH")
    if w.dtype != "bf16" or w.Lq < 64:
        return False
    if env in ("dense", "gather"):
        return env == "dense"
    tiles = causal_tiles(w.Lq, w.Lkv)
    per_tile = 2600.0 if (w.Hq // w.Hkv) % 2 == 0 else 4000.0
    dense_s = tiles * w.Hq * w.B * per_tile / (148.0 * 1.9e9)
    gather_s = (sum_min(w, w.topk) + sum_min(w, w.window)) * w.Hkv * w.B * 512.0 / 12.0e12
    return dense_s < gather_s


# ------------------------------------------------------------------- ours

def bench_ours(args, w, ws_, rank, local):
    import hybrid_sparse_attention_tcgen05_b200 as hs
    from hybrid_sparse_attention_tcgen05_b200 import inputs as gen

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_kind = load_peaks()
    l2 = measure_l2(dev)
    inp = gen.make_inputs(w, seed=args.seed + rank, device=str(dev))
    q, k, v = inp["q"], inp["k"], inp["v"]
    qs, gates = inp["q_sparse"], inp["gate"]
    shape = hs.shape_of(q, k)
    # rows scored per chunk: an 8 GiB f32 score buffer (8192 rows at 32k and 64k keys) keeps the
    # full layer's grids wide enough to fill the SMs (2 GiB chunks measured slower at both)
    chunk = args.row_chunk if args.row_chunk > 0 else min(w.Lq, max(1, (1 << 33) // (4 * w.Hkv * w.B * w.Lkv)))
    chunk = min(chunk, w.Lq)
    n_chunks = math.ceil(w.Lq / chunk)
    out = torch.empty_like(q)
    lse = torch.empty(w.B, w.Hq, w.Lq, dtype=torch.float32, device=dev)
    idx = torch.empty(w.B, w.Hkv, w.Lq, w.topk, dtype=torch.int32, device=dev)
    scores = torch.empty(w.B, w.Hkv, chunk, w.Lkv, dtype=torch.float32, device=dev)
    outs = [torch.empty_like(x) for x in qs]
    ws_full = hs.alloc_workspace(shape, w.topk, w.window, w.n_sparse, chunk, dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        # ev: list of events to record between stages (full+topk per chunk, sparse per layer)
        for c in range(n_chunks):
            r0 = c * chunk
            rc = min(chunk, w.Lq - r0)
            hs.full_attn_scores(q, k, v, row_begin=r0, row_count=rc, out=out, lse=lse,
                                scores=scores[:, :, :rc] if rc == chunk else
                                scores.view(-1)[: w.B * w.Hkv * rc * w.Lkv].view(w.B, w.Hkv, rc, w.Lkv),
                                ws=ws_full)
            if ev is not None:
                ev["full"].append(torch.cuda.Event(enable_timing=True))
                ev["full"][-1].record(stream)
            hs.topk(shape, scores[:, :, :rc] if rc == chunk else
                    scores.view(-1)[: w.B * w.Hkv * rc * w.Lkv].view(w.B, w.Hkv, rc, w.Lkv),
                    w.topk, row_begin=r0, idx=idx)
            if ev is not None:
                ev["topk"].append(torch.cuda.Event(enable_timing=True))
                ev["topk"][-1].record(stream)
        for n in range(w.n_sparse):
            hs.sparse_attn(qs[n], k, v, idx, gates[n], w.window, out=outs[n], ws=ws_full)
            if ev is not None:
                ev["sparse"].append(torch.cuda.Event(enable_timing=True))
                ev["sparse"][-1].record(stream)

    def block_step():
        # one hybrid block through the library's single call (hysparse_block)
        hs.block(q, k, v, qs, gates, w.topk, w.window, row_chunk=chunk, out_full=out, out_sparse=outs,
                 idx=idx, lse=lse, ws=ws_full)

    for _ in range(args.warmup):
        block_step()
        step()
    torch.cuda.synchronize()
    st = hs.workspace_status(ws_full)
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")

    # ---- timed region: K hybrid blocks, L2 flushed between them
    if ws_ > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    step_ms = []
    launches0 = hs.launch_count()
    with ClockSampler(local) as clk:
        t0 = time.perf_counter()
        for _ in range(args.steps):
            flush.fill_(1.0)          # evict L2 between timed steps
            e0 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            block_step()
            e1 = torch.cuda.Event(enable_timing=True)
            e1.record(stream)
            torch.cuda.synchronize()
            step_ms.append(e0.elapsed_time(e1))
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
    gpu_launches = hs.launch_count() - launches0
    if ws_ > 1:
        torch.distributed.barrier()
    total_ms = sum(step_ms)
    total_ms_max = max_over_ranks(total_ms, ws_, dev)
    ms_per_step = total_ms_max / args.steps
    tokens = w.B * w.Lq
    value = tokens * ws_ / (ms_per_step / 1e3)

    # ---- stage breakdown: the same work as separate C-ABI calls with CUDA
    # events between them on the launching stream (each sparse call rebuilds
    # its index bitmask, which the block call above builds once)
    stage_ms = {"full": 0.0, "topk": 0.0, "sparse": 0.0}
    for _ in range(args.steps):
        flush.fill_(1.0)
        ev = {"full": [], "topk": [], "sparse": []}
        e0 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step(ev)
        torch.cuda.synchronize()
        prev = e0
        seq = []
        for c in range(n_chunks):
            seq += [("full", ev["full"][c]), ("topk", ev["topk"][c])]
        seq += [("sparse", e) for e in ev["sparse"]]
        for name, e in seq:
            stage_ms[name] += prev.elapsed_time(e)
            prev = e
    # the full layer's forward alone (S1: no score pass), for its own tensor
    # rate beside the S1+S2 figure of the full stage (prefill only)
    fwd_ms = None
    if w.Lq > 1:
        fwd_ms = 0.0
        for _ in range(args.steps):
            flush.fill_(1.0)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for c in range(n_chunks):
                hs.full_attn_scores(q, k, v, want_scores=False, row_begin=c * chunk,
                                    row_count=min(chunk, w.Lq - c * chunk), out=out, lse=lse, ws=ws_full)
            e1.record(stream)
            torch.cuda.synchronize()
            fwd_ms += e0.elapsed_time(e1) / args.steps

    # ---- (--own-window) the sparse layers with their own window K/V: each
    # layer keeps [B, Lwin, Hkv, d] window keys and values (Lwin = Lkv in
    # prefill, where every position is projected; the window itself in
    # decode, a ring of the last tokens), timed against the same layers on
    # the shared cache, same index sets, L2 flushed before each timed pass
    own_window = None
    if getattr(args, "own_window", False):
        lwin = w.Lkv if w.Lq > 1 else min(w.window, w.Lkv)
        kvw = [gen.make_window_kv(w, lwin, seed=args.seed + 1000 + n, device=str(dev)) for n in range(w.n_sparse)]
        t_own = t_shared = 0.0
        for _ in range(args.steps):
            for own in (True, False):
                flush.fill_(1.0)
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for n in range(w.n_sparse):
                    kw_, vw_ = kvw[n] if own else (None, None)
                    hs.sparse_attn(qs[n], k, v, idx, gates[n], w.window, out=outs[n], ws=ws_full,
                                   k_win=kw_, v_win=vw_)
                e1.record(stream)
                torch.cuda.synchronize()
                if own:
                    t_own += e0.elapsed_time(e1) / args.steps / max(1, w.n_sparse)
                else:
                    t_shared += e0.elapsed_time(e1) / args.steps / max(1, w.n_sparse)
        if hs.workspace_status(ws_full) != 0:
            raise RuntimeError("device status after the own-window layers")
        own_window = {"lwin": lwin, "sparse_per_layer_ms": t_own, "shared_cache_per_layer_ms": t_shared,
                      "window_kv_bytes_per_layer": 2 * kvw[0][0].numel() * kvw[0][0].element_size(),
                      "api": "hybrid_sparse_attention_tcgen05_b200.sparse_attn(k_win=, v_win=) "
                             "(hysparse_sparse_attn_own_window)"}
        del kvw

    # ---- end to end through the public API with host buffers
    # Each step copies its inputs from pinned host memory, runs the block and
    # copies every output back.  Consecutive steps are pipelined the way a
    # serving loop would run them: host-to-device copies, the block and
    # device-to-host copies on three streams, device and host buffers double
    # buffered, so step s+1's inputs travel while step s computes and step
    # s-1's outputs travel back.  The timed region spans the first copy in to
    # the last copy out.
    # A decode step (one new query per sequence) brings only that token's
    # inputs: its queries and gates and its K/V row, appended to a KV cache
    # that stays on the device; a prefill step brings its whole prompt's Q/K/V.
    pin = lambda x: x.to("cpu").pin_memory()
    decode = w.Lq == 1
    kv_src = [k[:, -1:].contiguous(), v[:, -1:].contiguous()] if decode else [k, v]
    # one pinned host set serves both pipeline slots: the inputs are the same
    # every step (copies only read them), and the copies out run in order on
    # one stream, so no result buffer is written while an earlier copy into it
    # is in flight (halves the pinned host memory: 22 GB per rank at moe64k)
    h_in_set = [pin(x) for x in [q, *kv_src, *qs, *gates]]
    h_res_set = [torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(1 + len(qs))]
    h_in = [h_in_set, h_in_set]
    h_res = [h_res_set, h_res_set]
    if decode:
        caches = [(k.clone(), v.clone()) for _ in range(2)]   # resident caches (filled outside the timing)
        d_in = [[torch.empty_like(q), caches[i][0][:, -1:], caches[i][1][:, -1:],
                 *[torch.empty_like(x) for x in [*qs, *gates]]] for i in range(2)]
        d_kv = [caches[i] for i in range(2)]
    else:
        d_in = [[torch.empty_like(x) for x in [q, k, v, *qs, *gates]] for _ in range(2)]
        d_kv = [(d_in[i][1], d_in[i][2]) for i in range(2)]
    d_res = [[torch.empty_like(q) for _ in range(1 + len(qs))] for _ in range(2)]
    h2d = sum(x.numel() * x.element_size() for x in h_in[0])
    d2h = sum(x.numel() * x.element_size() for x in h_res[0])
    s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for e_ in comp_done + out_done:
        e_.record(stream)
    n_in = 3 + len(qs)

    def e2e_step(s_):
        i_ = s_ % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(comp_done[i_])          # step s-2 has finished reading these inputs
            for a_, b_ in zip(d_in[i_], h_in[i_]):
                a_.copy_(b_, non_blocking=True)
            in_done[i_].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(in_done[i_])
            s_comp.wait_event(out_done[i_])         # step s-2's outputs have left these buffers
            dq, (dk, dv) = d_in[i_][0], d_kv[i_]
            of, _, _, os_ = hs.block(dq, dk, dv, d_in[i_][3:n_in], d_in[i_][n_in:], w.topk, w.window,
                                     row_chunk=chunk, out_full=d_res[i_][0], out_sparse=d_res[i_][1:],
                                     idx=idx, lse=lse, ws=ws_full)
            comp_done[i_].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[i_])
            for a_, b_ in zip(h_res[i_], [of, *os_]):
                a_.copy_(b_, non_blocking=True)
            out_done[i_].record(s_out)

    # A prefill step moves gigabytes each way, so its layers are overlapped
    # with the copies one by one through the per-stage calls: the full layer
    # starts once Q, K and V have landed, sparse layer n once its queries and
    # gates have, and each layer's output leaves as soon as it is written.
    # (hysparse_block waits for every input and releases every output at
    # once; at moe64k that added the first step's whole copy in and the last
    # step's whole copy out to the timed region.)
    n_out = 1 + len(qs)
    if not decode:
        lay_in = [[ev() for _ in range(n_in - 3)] for _ in range(2)]      # Q, K, V first, then per layer
        lay_done = [[ev() for _ in range(n_out)] for _ in range(2)]
        lay_out = [[ev() for _ in range(n_out)] for _ in range(2)]
        for i_ in range(2):
            for e_ in lay_out[i_]:
                e_.record(stream)

        def e2e_step(s_):
            i_ = s_ % 2
            hin, din = h_in[i_], d_in[i_]
            with torch.cuda.stream(s_in):
                s_in.wait_event(comp_done[i_])      # step s-2 has finished reading these inputs
                for a_, b_ in zip(din[:3], hin[:3]):
                    a_.copy_(b_, non_blocking=True)
                in_done[i_].record(s_in)
                for n in range(n_in - 3):          # layer n's queries and gates
                    for a_, b_ in ((din[3 + n], hin[3 + n]), (din[n_in + n], hin[n_in + n])):
                        a_.copy_(b_, non_blocking=True)
                    lay_in[i_][n].record(s_in)
            with torch.cuda.stream(s_comp):
                dq, dk, dv = din[0], din[1], din[2]
                s_comp.wait_event(in_done[i_])
                s_comp.wait_event(lay_out[i_][0])   # step s-2's full output has left
                for c in range(n_chunks):
                    r0 = c * chunk
                    rc = min(chunk, w.Lq - r0)
                    sc_ = scores[:, :, :rc] if rc == chunk else \
                        scores.view(-1)[: w.B * w.Hkv * rc * w.Lkv].view(w.B, w.Hkv, rc, w.Lkv)
                    hs.full_attn_scores(dq, dk, dv, row_begin=r0, row_count=rc, out=d_res[i_][0], lse=lse,
                                        scores=sc_, ws=ws_full)
                    hs.topk(shape, sc_, w.topk, row_begin=r0, idx=idx)
                lay_done[i_][0].record(s_comp)
                for n in range(n_in - 3):
                    s_comp.wait_event(lay_in[i_][n])
                    s_comp.wait_event(lay_out[i_][1 + n])
                    hs.sparse_attn(din[3 + n], dk, dv, idx, din[n_in + n], w.window, out=d_res[i_][1 + n],
                                   ws=ws_full)
                    lay_done[i_][1 + n].record(s_comp)
                comp_done[i_].record(s_comp)
            with torch.cuda.stream(s_out):
                for n in range(n_out):
                    s_out.wait_event(lay_done[i_][n])
                    h_res[i_][n].copy_(d_res[i_][n], non_blocking=True)
                    lay_out[i_][n].record(s_out)
                out_done[i_].record(s_out)

    # enough steps that the pipeline's fill and drain (the first copy in
    # before any compute, the last compute and copy out after the last copy
    # in) are a small share of the timed region: about 6 s of device time,
    # 4 to 64 steps (ms_per_step is already the max over ranks, so every rank
    # runs the same count).  At moe64k one step's copies take ~0.2 s each way
    # against 0.35 s of compute, so over 4 steps the fill and drain alone
    # added a quarter to every step.
    e2e_steps = e2e_step_count(ms_per_step)
    e2e_step(0)
    e2e_step(1)
    torch.cuda.synchronize()
    if ws_ > 1:
        torch.distributed.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for s_ in range(e2e_steps):
        e2e_step(s_)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms_max = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, ws_, dev)
    e2e_value = tokens * ws_ / (e2e_ms_max / 1e3)

    # ---- roofline of the dominant stage
    wm = work_model(w)
    sparse_dense = sparse_path_is_dense(w)
    per = {kk: vv / args.steps for kk, vv in stage_ms.items()}
    dom = max(per, key=per.get)
    if dom == "full" and w.Lq == 1:
        # decode: one new row per sequence streams the whole cache -> HBM bound
        launches = n_chunks
        dur_s = per["full"] / launches / 1e3
        achieved = wm["kv_bytes"] / dur_s / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"kernel": "decode_full_mma+decode_combine", "bound": "hbm", "unit": "GB/s",
                "work": "K and V of every (batch, KV head) read once: 2*B*Lkv*Hkv*d*2 bytes"}
        key, srcs = "decode_full", ("sparse_mma.cu",)
    elif dom == "full":
        launches = n_chunks
        dur_s = per["full"] / launches / 1e3
        achieved = wm["flops_full_scores"] / n_chunks / dur_s / 1e12
        peak = peaks["bf16_tflops"]
        roof = {"kernel": "full_attn_scores", "bound": "tensor", "unit": "TFLOP/s",
                "work": "6*d*Hq per causal pair (QK^T+PV forward, QK^T score pass)"}
        key, srcs = "full_attn_scores", ("attn_tc.cu", "tc_attn.cuh", "tc_util.cuh")
    elif dom == "topk":
        launches = n_chunks
        dur_s = per["topk"] / launches / 1e3
        achieved = (wm["score_bytes"] / 2 + 4.0 * w.B * w.Hkv * w.Lq * w.topk) / n_chunks / dur_s / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"kernel": "topk", "bound": "hbm", "unit": "GB/s",
                "work": "4 B per causal (row, key, kv head) read + 4 B per index written"}
        key, srcs = "topk", ("topk.cu",)
    elif sparse_dense:
        # dense-masked tensor-core pass: report the method's useful FLOPs
        # against the tensor peak; the executed (all causal tiles) rate beside it
        launches = w.n_sparse
        dur_s = per["sparse"] / launches / 1e3
        useful = 4.0 * w.d * w.Hq * w.B * float(wm["keff"] + wm["weff"])
        achieved = useful / dur_s / 1e12
        peak = peaks["bf16_tflops"]
        roof = {"kernel": "sparse_attn (dense-masked: attn_fwd_tc<WIN> + attn_fwd_tc<SEL>)",
                "bound": "tensor", "unit": "TFLOP/s",
                "work": "4*d*Hq*(k_eff + w_eff) per row: the FLOPs the method needs",
                "executed_tflops": wm["flops_full_fwd"] / dur_s / 1e12}
        key, srcs = "sparse_pair", ("attn_tc.cu", "sparse_tc.cu", "tc_attn.cuh", "tc_util.cuh")
    else:
        launches = w.n_sparse
        dur_s = per["sparse"] / launches / 1e3
        achieved = wm["gather_bytes_per_layer"] / dur_s / 1e9
        if l2_served(w) and l2 is not None:
            # one KV head's K and V fit in L2 and the kernel walks the items KV
            # head by KV head: the gathered rows are L2 hits, rated against the
            # measured L2 read bandwidth
            peak = l2["peak_gbs"]
            bound, peak_src = "l2", "measured L2 read bandwidth (library probe, this run)"
        else:
            peak = peaks["hbm_gbs"]
            bound, peak_src = "hbm", None
        roof = {"kernel": "sparse_attn (gather: sparse_attn_mma)", "bound": bound, "unit": "GB/s",
                "work": "(k_eff + w_eff) K and V rows per (row, kv head) + q, gate, out, idx"}
        if peak_src:
            roof["peak_source"] = peak_src
        key, srcs = "sparse_attn", SPARSE_GATHER_SRCS
    roof.update({"achieved": achieved, "peak": peak,
                 "peak_kind": "measured (L2 probe)" if roof["bound"] == "l2" else f"{peak_kind} (burst)",
                 "frac": achieved / peak, "launch_ms": dur_s * 1e3,
                 "traffic": read_traffic(f"{w.name}/{key}", source_hash(*srcs))})
    stage_ctx = {
        "full": {"ms": per["full"], "tflops": (wm["flops_full_scores"] / (per["full"] / 1e3) / 1e12) if w.Lq > 1 else None,
                 "frac_of_peak": (wm["flops_full_scores"] / (per["full"] / 1e3) / 1e12 / peaks["bf16_tflops"])
                 if w.Lq > 1 else None,
                 "work": "6*d*Hq per causal pair (forward QK^T + PV, score-pass QK^T)" if w.Lq > 1 else None,
                 "hbm_gbs": (wm["kv_bytes"] / (per["full"] / 1e3) / 1e9) if w.Lq == 1 else None},
        "full_forward_only": ({"ms": fwd_ms, "tflops": wm["flops_full_fwd"] / (fwd_ms / 1e3) / 1e12,
                               "frac_of_peak": wm["flops_full_fwd"] / (fwd_ms / 1e3) / 1e12 / peaks["bf16_tflops"],
                               "work": "4*d*Hq per causal pair (QK^T + PV)"} if fwd_ms else None),
        "topk": {"ms": per["topk"], "gbs": (wm["score_bytes"] / 2 + 4.0 * w.B * w.Hkv * w.Lq * w.topk)
                 / (per["topk"] / 1e3) / 1e9},
        "sparse_per_layer": {"ms": per["sparse"] / max(1, w.n_sparse),
                             "path": "dense-masked" if sparse_dense else "gather",
                             "gbs": wm["gather_bytes_per_layer"] / (per["sparse"] / max(1, w.n_sparse) / 1e3) / 1e9},
    }
    sp_gbs = stage_ctx["sparse_per_layer"]["gbs"]
    if l2_served(w):
        stage_ctx["sparse_per_layer"]["frac_of_l2"] = sp_gbs / l2["peak_gbs"]
    else:
        stage_ctx["sparse_per_layer"]["frac_of_hbm"] = sp_gbs / peaks["hbm_gbs"]
    res = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded, generated on device)",
        "config": {"workload": w.name, "B": w.B, "Lq": w.Lq, "Lkv": w.Lkv, "Hq": w.Hq,
                   "Hkv": w.Hkv, "d": w.d, "topk": w.topk, "window": w.window,
                   "n_sparse": w.n_sparse, "row_chunk": chunk, "value_recipe": w.dist,
                   "l2": "flushed: 252 MiB written between timed steps",
                   "parallelism": f"replicas x{ws_}"},
        "clocks": clk.summary(),
        "e2e": {"value": e2e_value, "unit": "tokens/s", "ms_per_step": e2e_ms_max,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": ("hybrid_sparse_attention_tcgen05_b200.block; pinned host buffers; copy in, block, copy out "
                        "pipelined over three streams (device buffers double-buffered)") if w.Lq == 1 else
                       ("hybrid_sparse_attention_tcgen05_b200 full_attn_scores / topk / sparse_attn; pinned host "
                        "buffers; copies in and out overlapped layer by layer with the compute over three streams "
                        "(device buffers double-buffered)"),
                "steps": e2e_steps},
        "gpu_launches": gpu_launches,
        "roofline": roof,
        "stages_ms_per_step": per,
        "stages": stage_ctx,
        "l2_probe": l2,
        "wall_s_timed": wall,
    }
    if w.Lq == 1:
        res["decode_step_us"] = ms_per_step * 1e3
        if w.dtype == "bf16" and w.n_sparse > 1 and os.environ.get("HYSPARSE_LAYER_GROUP") != "0":
            # the stage loop times the sparse layers as single-layer calls;
            # hysparse_block runs them as one grouped launch, whose time is the
            # step less the other two stages
            res["sparse_grouped_ms_est"] = max(0.0, ms_per_step - per["full"] - per["topk"])
            res["stages_note"] = ("stages time each sparse layer as its own call; the block runs the "
                                  "decode sparse layers as one grouped launch (sparse_grouped_ms_est)")
    if own_window is not None:
        res["own_window"] = own_window
    res["_inputs"] = inp
    return res


# ------------------------------------------------- decode, mixed lengths

def bench_varlen(args, w, ws_, rank, local):
    """Decode with every sequence at its own cache length (seeded, uniform in
    [window, Lkv]) through hysparse_block_varlen.  Same timing rules as the
    fixed-length run; the roofline is the whole block against HBM."""
    import hybrid_sparse_attention_tcgen05_b200 as hs
    from hybrid_sparse_attention_tcgen05_b200 import inputs as gen

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_kind = load_peaks()
    inp = gen.make_inputs(w, seed=args.seed + rank, device=str(dev))
    q, k, v = inp["q"], inp["k"], inp["v"]
    qs, gates = inp["q_sparse"], inp["gate"]
    g = torch.Generator().manual_seed(args.seed + 1000 + rank)
    lens = torch.randint(w.window, w.Lkv + 1, (w.B,), generator=g).to(torch.int32)
    kv_len = lens.to(dev)
    shape = hs.shape_of(q, k)
    ws_full = hs.alloc_workspace(shape, w.topk, w.window, w.n_sparse, 1, dev)
    out = torch.empty_like(q)
    outs = [torch.empty_like(x) for x in qs]
    lse = torch.empty(w.B, w.Hq, 1, dtype=torch.float32, device=dev)
    idx = torch.empty(w.B, w.Hkv, 1, w.topk, dtype=torch.int32, device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    P = args.page_size
    if P > 0:
        # paged caches: every sequence's pages scattered over a shuffled pool
        if P & (P - 1):
            raise SystemExit("--page-size must be a power of two")
        max_pages = (w.Lkv + P - 1) // P
        need = [(int(x) + P - 1) // P for x in lens]
        perm = torch.randperm(sum(need), generator=g).tolist()
        table_h = torch.full((w.B, max_pages), -1, dtype=torch.int32)
        kp = torch.zeros(sum(need), P, w.Hkv, w.d, dtype=k.dtype, device=dev)
        vp = torch.zeros_like(kp)
        nxt = 0
        for b_ in range(w.B):
            for pg in range(need[b_]):
                page = perm[nxt]
                nxt += 1
                table_h[b_, pg] = page
                lo_, hi_ = pg * P, min(int(lens[b_]), (pg + 1) * P)
                kp[page, : hi_ - lo_] = k[b_, lo_:hi_]
                vp[page, : hi_ - lo_] = v[b_, lo_:hi_]
        table = table_h.to(dev)

    def run_block(qq, qq_s, gg):
        if P > 0:
            hs.block_paged(qq, kp, vp, qq_s, gg, w.topk, w.window, kv_len, table, max_len=w.Lkv, out_full=out,
                           out_sparse=outs, idx=idx, lse=lse, ws=ws_full)
        else:
            hs.block(qq, k, v, qq_s, gg, w.topk, w.window, out_full=out, out_sparse=outs, idx=idx, lse=lse,
                     ws=ws_full, kv_len=kv_len)

    def block_step():
        run_block(q, qs, gates)

    for _ in range(args.warmup):
        block_step()
    torch.cuda.synchronize()
    st = hs.workspace_status(ws_full)
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    if ws_ > 1:
        torch.distributed.barrier()
    step_ms = []
    launches0 = hs.launch_count()
    with ClockSampler(local) as clk:
        t0 = time.perf_counter()
        for _ in range(args.steps):
            flush.fill_(1.0)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            block_step()
            e1.record(stream)
            torch.cuda.synchronize()
            step_ms.append(e0.elapsed_time(e1))
        wall = time.perf_counter() - t0
    gpu_launches = hs.launch_count() - launches0
    if ws_ > 1:
        torch.distributed.barrier()
    ms_per_step = max_over_ranks(sum(step_ms), ws_, dev) / args.steps
    value = w.B * ws_ / (ms_per_step / 1e3)

    # end to end: each step brings the new token's queries, gates and K/V row
    # from pinned host memory, writes the K/V row into each sequence's cache
    # at its own position, runs the block and reads every output back
    pin = lambda x: x.to("cpu").pin_memory()
    rows = torch.arange(w.B, device=dev)
    pos = kv_len.long() - 1
    h_in = [pin(x) for x in [q, k[rows, pos].unsqueeze(1), v[rows, pos].unsqueeze(1), *qs, *gates]]
    d_in = [torch.empty_like(x, device=dev) for x in h_in]
    h_res = [torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(1 + len(qs))]
    h2d = sum(x.numel() * x.element_size() for x in h_in)
    d2h = sum(x.numel() * x.element_size() for x in h_res)
    n_in = 3 + len(qs)

    if P > 0:   # where each sequence's new row lives in the page pool
        prow = table[rows, pos // P].long()
        pcol = pos % P

    def e2e_step():
        for a_, b_ in zip(d_in, h_in):
            a_.copy_(b_, non_blocking=True)
        if P > 0:
            kp[prow, pcol] = d_in[1][:, 0]
            vp[prow, pcol] = d_in[2][:, 0]
        else:
            k[rows, pos] = d_in[1][:, 0]
            v[rows, pos] = d_in[2][:, 0]
        run_block(d_in[0], d_in[3:n_in], d_in[n_in:])
        for a_, b_ in zip(h_res, [out, *outs]):
            a_.copy_(b_, non_blocking=True)

    e2e_steps = e2e_step_count(ms_per_step)
    e2e_step()
    torch.cuda.synchronize()
    if ws_ > 1:
        torch.distributed.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, ws_, dev)

    # algorithmic HBM bytes of the block: every sequence's K and V read once by
    # the full layer, then each sparse layer's gathered rows
    L = lens.double()
    esz = 2
    kv_bytes = float((2 * L * w.Hkv * w.d * esz).sum())
    gather = float(((torch.clamp(L, max=w.topk) + torch.clamp(L, max=w.window)) * w.Hkv * 2 * w.d * esz).sum())
    bytes_total = kv_bytes + w.n_sparse * gather
    achieved = bytes_total / (ms_per_step / 1e3) / 1e9
    roof = {"kernel": ("hysparse_block_paged" if P > 0 else "hysparse_block_varlen")
                      + " (decode_full_mma + decode_combine + topk + n x sparse_attn_mma)",
            "bound": "hbm", "unit": "GB/s",
            "work": "each sequence's K and V read once (2*L_b*Hkv*d*2 B) + per sparse layer its gathered "
                    "(min(k, L_b) + min(w, L_b)) K and V rows",
            "achieved": achieved, "peak": peaks["hbm_gbs"], "peak_kind": f"{peak_kind} (burst)",
            "frac": achieved / peaks["hbm_gbs"], "launch_ms": ms_per_step, "traffic": None}
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded, generated on device)",
        "config": {"workload": f"{w.name}-varlen" + (f"-paged{P}" if P > 0 else ""), "B": w.B, "Lq": 1,
                   "Lkv_max": w.Lkv, "Hq": w.Hq, "page_size": P if P > 0 else None,
                   "Hkv": w.Hkv, "d": w.d, "topk": w.topk, "window": w.window, "n_sparse": w.n_sparse,
                   "kv_len": {"min": int(lens.min()), "mean": float(L.mean()), "max": int(lens.max()),
                              "draw": f"uniform in [{w.window}, {w.Lkv}], seed {args.seed + 1000 + rank}"},
                   "l2": "flushed: 252 MiB written between timed steps", "parallelism": f"replicas x{ws_}"},
        "clocks": clk.summary(),
        "e2e": {"value": w.B * ws_ / (e2e_ms / 1e3), "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": "hybrid_sparse_attention_tcgen05_b200.block(kv_len=...); pinned host buffers; copy in, "
                       "K/V row into each cache at its position, block, copy out, one stream",
                "steps": e2e_steps},
        "gpu_launches": gpu_launches,
        "roofline": roof,
        "decode_step_us": ms_per_step * 1e3,
        "wall_s_timed": wall,
    }


# --------------------------------------------------------- CPU (oracle) arm

def row_cost(w, i):
    """Oracle cost of one query row (per batch element), in multiply-adds:
    full layer Hq*(pos+1)*2d, each sparse layer Hq*(k_eff+w_eff)*2d."""
    pos = w.Lkv - w.Lq + i
    n = pos + 1
    return w.Hq * 2 * w.d * (n + w.n_sparse * (min(n, w.topk) + min(n, w.window)))


def total_cost(w):
    off = w.Lkv - w.Lq
    full = w.Hq * 2 * w.d * (w.Lq * (off + 1) + w.Lq * (w.Lq - 1) // 2)
    sp = w.Hq * 2 * w.d * w.n_sparse * (sum_min(w, w.topk) + sum_min(w, w.window))
    return float(full + sp) * w.B


def oracle_inputs(w, seed, dev_inputs=None):
    """Batch element 0 of the workload's inputs on the host: (k, v, q,
    q_sparse, gate), widened exactly to fp32.  Uses the device tensors when
    given (same seed, so the same values the GPU timed), else draws on the
    CPU when small enough, else on the GPU."""
    from hybrid_sparse_attention_tcgen05_b200 import inputs as gen
    if dev_inputs is None:
        small = w.Lq * w.Hq * w.d * (1 + w.n_sparse) * w.B <= (1 << 28) and \
            w.B * w.Lkv * w.Hkv * w.d <= (1 << 27)
        dev_inputs = gen.make_inputs(w, seed=seed, device="cpu" if small or not torch.cuda.is_available()
                                     else "cuda")
    f = lambda t: t[0:1].to("cpu", torch.float32)
    return (f(dev_inputs["k"]), f(dev_inputs["v"]), f(dev_inputs["q"]),
            [f(x) for x in dev_inputs["q_sparse"]], [f(x) for x in dev_inputs["gate"]])


def oracle_sample_time(w, seed, budget_s, host=None):
    """Time oracle.block_rows on a row sample sized to ~budget_s; returns
    (extrapolated seconds for the whole workload, sample description,
    threads, sample seconds)."""
    import oracle

    threads = len(os.sched_getaffinity(0))
    oracle.set_threads(threads)
    k_h, v_h, q_h, qs_h, g_h = host
    w1 = w.with_(B=1)
    scale = 1.0 / math.sqrt(w.d)

    def run(rows_i):
        rows = [(0, i) for i in rows_i]
        qr = q_h[0, rows_i]
        qsr = torch.stack([x[0, rows_i] for x in qs_h])
        gr = torch.stack([x[0, rows_i] for x in g_h])
        t0 = time.perf_counter()
        oracle.block_rows(qr, k_h, v_h, rows, w1.Lq, scale, qsr, gr, w.topk, w.window)
        return time.perf_counter() - t0

    # calibrate on a few of the costliest rows (the last ones)
    probe = list(range(max(0, w1.Lq - 2), w1.Lq))
    tp = run(probe)
    rate = sum(row_cost(w1, i) for i in probe) / max(tp, 1e-6)         # units / s
    per_row_avg = total_cost(w1) / w1.Lq
    n = int(max(1, min(w1.Lq, rate * budget_s / per_row_avg)))
    stride = w1.Lq / n
    rows_i = sorted(set(min(w1.Lq - 1, int(j * stride + stride / 2)) for j in range(n)))
    ts = run(rows_i)
    units = sum(row_cost(w1, i) for i in rows_i)
    est = ts * total_cost(w) / units
    desc = (f"{len(rows_i)} evenly spaced query rows of {w1.Lq} (batch element 0 of {w.B}), all "
            f"heads, full layer + top-k + {w.n_sparse} sparse layers, {ts:.1f} s of oracle time; "
            f"extrapolated to the whole workload by the exact per-row cost (pos+1 keys in the full "
            f"layer, k_eff+w_eff per sparse layer)")
    return est, desc, threads, ts


def bench_reference(args, w):
    host = oracle_inputs(w, args.seed)
    per = args.cpu_budget / max(1, args.steps + args.warmup)
    for _ in range(args.warmup):
        oracle_sample_time(w, args.seed, per, host)
    vals, sample_s = [], []
    desc, threads = "", 1
    for _ in range(max(1, args.steps)):
        e, desc, threads, ts = oracle_sample_time(w, args.seed, per, host)
        vals.append(e)
        sample_s.append(ts)
    est = statistics.median(vals)
    tokens = w.B * w.Lq
    value = tokens / est
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": est * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "impl": "reference",
        "config": {"workload": w.name, "B": w.B, "Lq": w.Lq, "Lkv": w.Lkv, "Hq": w.Hq,
                   "Hkv": w.Hkv, "d": w.d, "topk": w.topk, "window": w.window,
                   "n_sparse": w.n_sparse},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        # each step times a row sample, not the whole workload: ms_per_step is
        # the whole workload's time extrapolated from that sample
        "extrapolated": True,
        "sample_s_per_step": statistics.median(sample_s),
        "sample_s_total": sum(sample_s),
    }


def decode_summary(res, peaks):
    """The decode step's figures for the headline line: step latency, tokens/s
    (device and end to end), per-stage times, and the sparse gather stage's
    achieved HBM bandwidth against the measured HBM peak."""
    st = res["stages"]
    sp = st["sparse_per_layer"]
    return {"workload": res["config"]["workload"], "config": res["config"],
            "decode_step_us": res["ms_per_step"] * 1e3, "value": res["value"], "unit": res["unit"],
            "e2e": res["e2e"], "gpu_launches": res["gpu_launches"], "clocks": res["clocks"],
            "stages_ms_per_step": res["stages_ms_per_step"],
            "full": {"ms": st["full"]["ms"], "hbm_gbs": st["full"]["hbm_gbs"],
                     "frac_of_hbm": st["full"]["hbm_gbs"] / peaks["hbm_gbs"]},
            "sparse_gather": {"ms_per_layer": sp["ms"], "hbm_gbs": sp["gbs"],
                              "frac_of_hbm": sp["gbs"] / peaks["hbm_gbs"], "peak_gbs": peaks["hbm_gbs"],
                              "work": "(k_eff + w_eff) K and V rows per (sequence, kv head) + q, gate, "
                                      "out, idx"},
            "roofline": res["roofline"], **({"own_window": res["own_window"]} if "own_window" in res else {}),
            **({"sparse_grouped_ms_est": res["sparse_grouped_ms_est"], "stages_note": res["stages_note"]}
               if "sparse_grouped_ms_est" in res else {})}


def profile_stage(args, w):
    """A few launches of one stage on a small case, for ncu captures: the
    inputs and the index set are made first (one untimed block), then the
    stage's C-ABI call runs `--profile-reps` times."""
    import hybrid_sparse_attention_tcgen05_b200 as hs
    from hybrid_sparse_attention_tcgen05_b200 import inputs as gen
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = w.with_(n_sparse=1)
    inp = gen.make_inputs(w, seed=args.seed, device=str(dev))
    q, k, v = inp["q"], inp["k"], inp["v"]
    chunk = min(w.Lq, 4096)
    out, lse, idx, outs = hs.block(q, k, v, inp["q_sparse"], inp["gate"], w.topk, w.window, row_chunk=chunk)
    torch.cuda.synchronize()
    shape = hs.shape_of(q, k)
    ws = hs.alloc_workspace(shape, w.topk, w.window, 1, chunk, dev)
    for _ in range(args.profile_reps):
        if args.profile_stage == "sparse":
            hs.sparse_attn(inp["q_sparse"][0], k, v, idx, inp["gate"][0], w.window, out=outs[0], ws=ws)
        elif args.profile_stage == "full":
            hs.full_attn_scores(q, k, v, row_begin=w.Lq - chunk, row_count=chunk, out=out, lse=lse, ws=ws)
        else:
            sc = hs.full_attn_scores(q, k, v, row_begin=w.Lq - chunk, row_count=chunk, out=out, lse=lse,
                                     ws=ws)[2]
            hs.topk(shape, sc, w.topk, row_begin=w.Lq - chunk, idx=idx)
    torch.cuda.synchronize()
    if hs.workspace_status(ws) != 0:
        raise RuntimeError("device status set")
    print(json.dumps({"profile_stage": args.profile_stage, "workload": w.name, "reps": args.profile_reps}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="moe64k",
                    help="headline workload (default: the largest single-GPU configuration)")
    ap.add_argument("--no-decode", action="store_true",
                    help="prefill workloads: skip the decode step that the line also reports")
    ap.add_argument("--profile-stage", choices=["full", "topk", "sparse"], default=None,
                    help="run a few launches of one stage (for ncu) and exit; no timing")
    ap.add_argument("--profile-reps", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--row-chunk", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--own-window", action="store_true",
                    help="also time the sparse layers on their own window K/V against the shared cache")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work")
    ap.add_argument("--varlen", action="store_true",
                    help="decode workloads: every sequence at its own cache length (hysparse_block_varlen)")
    ap.add_argument("--page-size", type=int, default=0,
                    help="with --varlen: paged caches of this many rows per page (hysparse_block_paged)")
    ap.add_argument("--seq", type=int, default=0,
                    help="override the cache length (and the prefill length) for small profiling runs")
    args = ap.parse_args()

    from hybrid_sparse_attention_tcgen05_b200 import inputs as gen
    w = gen.WORKLOADS[args.workload]
    if args.seq > 0:
        w = w.with_(Lkv=args.seq, Lq=1 if w.Lq == 1 else args.seq, name=f"{w.name}@{args.seq}")
    world, rank, local = dist_env()

    if args.profile_stage:
        profile_stage(args, w)
        return 0

    if args.impl == "reference":
        if rank != 0:
            return 0
        res = bench_reference(args, w)
        print(json.dumps(res), flush=True)
        return 0

    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    try:
        if args.varlen:
            if w.Lq != 1:
                raise SystemExit("--varlen applies to decode workloads (Lq = 1)")
            res = bench_varlen(args, w, world, rank, local)
            if rank == 0:
                print(json.dumps(res), flush=True)
            return 0
        res = bench_ours(args, w, world, rank, local)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            host = oracle_inputs(w, args.seed, res.pop("_inputs"))
            est, desc, threads, _ = oracle_sample_time(w, args.seed, args.cpu_budget, host)
            res["cpu_baseline"] = {"value": w.B * w.Lq / est, "unit": "tokens/s", "cores": threads,
                                   "kind": "oracle", "sample": desc}
        res.pop("_inputs", None)
        if w.Lq > 1 and not args.no_decode and args.seq == 0:
            # the decode step of the same line (64 sequences, 32768-token caches)
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
            dres = bench_ours(args, gen.WORKLOADS["decode"], world, rank, local)
            dres.pop("_inputs", None)
            res["decode"] = decode_summary(dres, load_peaks()[0])
            res["gpu_launches_decode"] = dres["gpu_launches"]
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
