"""Benchmark of the GQLA decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one decode step of the batch through the whole hot path: the
MQA-absorb path (gqla_absorb_query -> gqla_decode_absorb -> gqla_combine with
W_UV) and the GQA path (gqla_decode_gqa_step: the GQA decode, then the
combine for the sequences that span more than one chunk) over the same batch.
The two paths are independent, so the GQA path runs on a second stream beside
the absorb path's decode and combine (after the query absorption has started).
Both decodes fill the device on their own, so beside each other they would run
one after the other but for a lead in the absorb split plan
(gqla_decode_absorb_lead, planned by gqla_plan_lead from the calls' own
times, reported as "absorb_lead"): the absorb decode, launched first, has a few
chunks about twice as long as the rest on the CTAs that the SMs left idle by
the GQA decode's CTA count can hold, so the GQA decode starts on the SMs of
the short chunks while the long ones keep the rest busy.  --no-lead runs the
step with equal chunks.  The per-call ("per_kernel") and per-path times are
always taken with equal chunks.
The one-shot cache expansion (gqla_expand_cache) is a deploy-time conversion,
not part of a step; it is timed once and reported under "expand".

value   = decode tokens per second of the whole job: N ranks x batch x s_q
          tokens per step / (device time per step, max over ranks); each rank
          decodes its own batch (independent sequences, no collective on the
          data path: weak scaling).
e2e     = the same through the C ABI with host buffers: each step copies the
          queries, page table and lengths from pinned host memory and reads
          both paths' outputs back into pinned memory, inside the timed region
          (replayed as one CUDA graph).  The batch is cut into sub-batches of
          whole sequences ("sub_batches": their sizes; two equal ones from 8
          sequences up, or relative sizes from --e2e-parts such as 1,6,1), each
          a full step of its own with its own split plan, so one sub-batch's copies
          overlap another's kernels: inputs on a copy-in stream, the absorb
          path on the main stream, the GQA path on a second stream, outputs
          on a copy-out stream as soon as each path of a sub-batch is done.
Timing  = the step is captured into a CUDA graph; the K timed steps are issued
          back to back, each replay between two CUDA events on the stream
          (device time, no host launch overhead), with an L2 flush (a 256 MiB
          write, then a 256 MiB read so no dirty line is left) before every
          step, outside its events; one synchronize ends the timed region,
          while an NVML sampler records SM clocks and throttle reasons.  Each
          path's step ("per_path") is timed the same way from a graph of that
          path's calls alone; the per-call breakdown ("per_kernel") comes from a
          graph that runs the five calls in order on one stream with an event
          record around every call.  W >= 3 untimed eager and W graph warm-up
          steps come first.
workload: by default the largest single-GPU configuration of the suite
          (dsv3_h128_b64_l8192_mtp2: 128 heads, 8 groups, 64 sequences of
          8192 tokens, s_q = 2); at N = 1 every other workload of the suite
          follows under "workloads" (step time, per-call times, each path's
          roofline fractions), unless --headline-only.
--gpus N  one rank per GPU: under torchrun WORLD_SIZE must equal N; started
          without torchrun, the script relaunches itself as N ranks.
roofline: the dominant kernel's algorithmic bytes (or FLOPs) per launch over
          its mean event-timed duration, against MEASURED_PEAKS.json.
cpu_baseline: the fp64 CPU oracle on a bounded sample of the same workload
          (rank 0, N = 1 only).  --impl reference times the oracle alone.
"""
from __future__ import annotations

import argparse
import hashlib
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

# the largest single-GPU configuration of the suite: 64 sequences x 8192 tokens,
# two MTP query tokens (the absorb path is tensor-bound there)
DEFAULT_WORKLOAD = "dsv3_h128_b64_l8192_mtp2"
METRIC = "decode-attn tokens/s & µs/step per path; % of B200 HBM / tensor roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20

# Kernel source files whose ncu counters are stored in profiles/traffic.json;
# a stored figure is used only while the source hash still matches.
KERNEL_SOURCES = {
    "decode_gqa": ["decode_attention_06_b200/csrc/decode_gqa.cu",
                   "decode_attention_06_b200/csrc/sm100.cuh"],
    "decode_absorb": ["decode_attention_06_b200/csrc/decode_absorb.cu",
                      "decode_attention_06_b200/csrc/sm100.cuh"],
}


# ------------------------------------------------------------------ helpers

def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def _src_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _stored_traffic(kernel, workload, s_q):
    """ncu DRAM bytes per launch stored for (kernel, workload, s_q), or None when
    there is none or the kernel's source has changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p) or kernel not in KERNEL_SOURCES:
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel, {}).get(f"{workload}/sq{s_q}")
    if not e or e.get("source_hash") != _src_hash(KERNEL_SOURCES[kernel]):
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index, period_s=0.0002):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._period = period_s
        self._dev = device_index
        self._thread = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self._dev)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML missing: report no samples rather than guessing
            self._nvml = None
            return self
        self._started = threading.Event()
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        self._started.wait(0.5)  # the sampler runs before the timed work is issued
        return self

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM))
                r = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._started.set()
            time.sleep(self._period)

    def __exit__(self, *a):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": sorted(self.reasons - {"gpu_idle"})}


# ------------------------------------------------------------------ workload accounting

def accounting(w, case, s_q, num_splits):
    """Algorithmic bytes / FLOPs per launch (what the kernel must move / compute)."""
    seqlens = case["seqlens"].cpu().tolist()
    B, h, g = len(seqlens), w.num_heads, w.num_groups
    tokens = sum(seqlens)
    # visible (query, token) pairs: query s of a length-L sequence sees L - s_q + s + 1 tokens
    pairs = sum(max(0, L - s_q + s + 1) for L in seqlens for s in range(s_q))
    pages = [math.ceil(L / 64) for L in seqlens]
    T = sum(pages)
    k = math.ceil(T / num_splits) if T else 1
    pieces, start = 0, 0
    for n in pages:
        if n:
            pieces += (start + n - 1) // k - start // k + 1
        start += n
    rows = B * s_q * h
    gqa_tok = (2 * g * 128 + 64) * 2  # expanded bytes per token: 4224 at g = 8, 2176 at g = 4
    acc = {
        "decode_absorb": {
            "bytes": tokens * 1152 + rows * 576 * 2 + pieces * s_q * h * (512 + 1) * 4,
            "flops": 2.0 * h * pairs * (576 + 512),
        },
        "decode_gqa": {
            "bytes": tokens * gqa_tok + rows * 192 * 2 + pieces * s_q * h * (128 + 1) * 4,
            "flops": 2.0 * h * pairs * (192 + 128),
        },
        "absorb_query": {"bytes": rows * (192 + 576) * 2 + g * 512 * 128 * 2,
                         "flops": 2.0 * rows * 512 * 128},
        "combine_absorb": {"bytes": pieces * s_q * h * 513 * 4 + rows * 128 * 2 + g * 512 * 128 * 2,
                           "flops": 2.0 * rows * 512 * 128},
        "combine_gqa": {"bytes": pieces * s_q * h * 129 * 4 + rows * 128 * 2, "flops": 0.0},
        "expand": {"bytes": case["num_pages"] * 64 * (1152 + gqa_tok) + 2 * g * 512 * 128 * 2,
                   "flops": 2.0 * case["num_pages"] * 64 * 512 * 256 * g},
    }
    return acc, {"tokens": tokens, "pairs": pairs, "pieces": pieces}


# ------------------------------------------------------------------ CPU oracle timing

def _gather(case, batch_ids):
    """CPU copy of the chosen sequences with their pages only (for the oracle)."""
    ps = case["page_size"]
    pt = case["page_table"].cpu()
    sl = case["seqlens"].cpu()
    pages, rows = [], []
    for b in batch_ids:
        n = max(1, math.ceil(int(sl[b]) / ps))
        rows.append(list(range(len(pages), len(pages) + n)))
        pages.extend(pt[b, :n].tolist())
    dev = case["latent"].device
    latent = case["latent"][torch.tensor(pages, device=dev)].cpu()
    new_pt = torch.zeros(len(batch_ids), max(len(r) for r in rows), dtype=torch.int32)
    for i, r in enumerate(rows):
        new_pt[i, :len(r)] = torch.tensor(r, dtype=torch.int32)
    q = case["q"][torch.tensor(batch_ids, device=case["q"].device)].cpu()
    return q, latent, new_pt, sl[batch_ids].clone()


def cpu_oracle_rate(case, w, s_q, budget_s=10.0, unit_groups=None):
    """Run the oracle on successive sequences (all groups, or `unit_groups` of
    them) until budget_s has elapsed; return (tokens/s, cores, description)."""
    import oracle
    cores = oracle.num_threads()
    B = case["seqlens"].numel()
    per_call = max(1, cores // (unit_groups or w.num_groups))
    done_seqs, elapsed, b = 0, 0.0, 0
    while b < B and (elapsed < budget_s or done_seqs == 0):
        ids = list(range(b, min(B, b + per_call)))
        q, lat, pt, sl = _gather(case, ids)
        units = None
        if unit_groups:
            units = [(i, gi) for i in range(len(ids)) for gi in range(unit_groups)]
        t0 = time.perf_counter()
        oracle.decode(q, lat, pt, sl, case["w_uk"].cpu(), case["w_uv"].cpu(), w.num_groups,
                      units=units)
        elapsed += time.perf_counter() - t0
        done_seqs += len(ids)
        b += len(ids)
    frac = (unit_groups or w.num_groups) / w.num_groups
    rate = done_seqs * s_q * frac / elapsed
    what = (f"{done_seqs} of {B} sequences"
            + (f", {unit_groups} of {w.num_groups} groups" if unit_groups else ", all groups")
            + f", {elapsed:.1f} s fp64 oracle")
    return rate, cores, what


# ------------------------------------------------------------------ the GPU arm

_FLUSH = {}


def flush_l2(dev):
    """Write a buffer larger than L2, then read another one: the write evicts every
    line of the step's data, and the read makes L2 write the dirty lines of the first
    buffer back before the step starts, so their write-back does not land in the
    next timed kernel."""
    if dev not in _FLUSH:
        _FLUSH[dev] = (torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev),
                       torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev),
                       torch.empty((), dtype=torch.float32, device=dev))
    buf, rd, out = _FLUSH[dev]
    buf.fill_(1.0)
    torch.sum(rd, dim=0, out=out)


CALL_NAMES = ["absorb_query", "decode_absorb", "combine_absorb", "decode_gqa", "combine_gqa"]


class Workbench:
    """One workload (and s_q) on this rank's GPU: its seeded inputs, the expanded
    cache, both paths' buffers, and the five calls of a step through the C ABI."""

    def __init__(self, name, s_q, rank, dev, splits=None, lead=True):
        from decode_attention_06_b200 import gqla, synth
        self.gqla = gqla
        self.name, self.dev = name, dev
        self.w = w = synth.WORKLOADS[name]
        self.s_q = s_q = s_q or w.s_q[0]
        self.case = case = synth.make_case(w.num_heads, w.num_groups, w.seqlens(), s_q, paged=w.paged,
                                           seed=w.seed + 1000 * rank, device=str(dev))
        h, g = w.num_heads, w.num_groups
        self.B = case["seqlens"].numel()
        self.dims = dims = gqla.make_dims(h, g)
        self.kv = gqla.make_kv_index(case["page_table"], case["seqlens"], case["num_pages"])
        self.n_slots = case["num_pages"] * case["page_size"]
        # split counts planned on the host from the lengths (one wave at most, chunks
        # that hold two sequences' pieces counted at their cost)
        lens_host = case["seqlens"].cpu()
        self.splits = {"absorb": splits or gqla.plan_splits("absorb", h, s_q, lens_host),
                       "gqa": splits or gqla.plan_splits("gqa", h, s_q, lens_host, fused=True)}
        self.kvx = torch.empty(g, self.n_slots, 256, dtype=torch.bfloat16, device=dev)
        self.kr = torch.empty(self.n_slots, 64, dtype=torch.bfloat16, device=dev)
        self.ba = gqla.DecodeBuffers(dims, self.B, s_q, self.splits["absorb"], "absorb", device=dev)
        self.bg = gqla.DecodeBuffers(dims, self.B, s_q, self.splits["gqa"], "gqa", device=dev)
        self.gqa_stream = torch.cuda.Stream(device=dev)
        self.calls = self.make_calls(case["q"], self.kv)
        # the absorb split plan's lead chunks in the step (gqla_plan_lead, from the calls'
        # own times): (0, 16) = equal chunks
        self.lead = (0, 16)
        self.use_lead = lead
        self.e2e_lead = False
        self.call_ms = None

    def gqa_step_call(self, q, kv):
        """The GQA path as one call (gqla_decode_gqa_step: the decode, and the combine for
        the sequences that span more than one chunk)."""
        gqla, bg = self.gqla, self.bg
        return lambda: gqla.gqla_decode_gqa_step(self.dims, q, self.kvx, self.kr, kv, bg.num_splits,
                                                 bg.o_part, bg.lse_part, bg.out, bg.lse, bg.workspace)

    def launches_per_step(self):
        """Kernels one step launches: query absorption, absorb decode and combine; the GQA
        decode, and its combine unless every sequence lies in one chunk (one split)."""
        return 3 + 1 + (1 if self.splits["gqa"] > 1 else 0)

    def make_calls(self, q, kv):
        gqla, dims, case, ba, bg, s_q = self.gqla, self.dims, self.case, self.ba, self.bg, self.s_q
        return [
            lambda: gqla.gqla_absorb_query(dims, q, case["w_uk"], ba.q_absorbed),
            lambda: gqla.gqla_decode_absorb(dims, ba.q_absorbed, case["latent"], kv, ba.num_splits,
                                            ba.o_part, ba.lse_part, ba.workspace),
            lambda: gqla.gqla_combine(dims, kv, s_q, ba.num_splits, 512, ba.o_part, ba.lse_part,
                                      case["w_uv"], ba.out, ba.lse),
            lambda: gqla.gqla_decode_gqa(dims, q, self.kvx, self.kr, kv, bg.num_splits, bg.o_part,
                                         bg.lse_part, bg.workspace),
            lambda: gqla.gqla_combine(dims, kv, s_q, bg.num_splits, 128, bg.o_part, bg.lse_part,
                                      None, bg.out, bg.lse),
        ]

    def time_expand(self):
        """The one-shot expansion, timed on its own: the tensor-core version, then the
        bit-exact sequential-order one (whose output the steps use).  Returns ms."""
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c = self.case
        res = []
        for fn in (self.gqla.gqla_expand_cache_tc, self.gqla.gqla_expand_cache):
            fn(self.dims, c["latent"], c["w_uk"], c["w_uv"], self.kvx, self.kr)
            flush_l2(self.dev)
            e0.record()
            fn(self.dims, c["latent"], c["w_uk"], c["w_uv"], self.kvx, self.kr)
            e1.record()
            torch.cuda.synchronize()
            res.append(e0.elapsed_time(e1))
        return res[1], res[0]

    def lead_calls(self, q, kv, ba, lead):
        """The absorb decode and combine on a split plan with lead chunks."""
        gqla, dims, case = self.gqla, self.dims, self.case
        return (lambda: gqla.gqla_decode_absorb_lead(dims, ba.q_absorbed, case["latent"], kv, ba.num_splits,
                                                     lead[0], lead[1], ba.o_part, ba.lse_part, ba.workspace),
                lambda: gqla.gqla_combine_lead(dims, kv, self.s_q, ba.num_splits, lead[0], lead[1], 512,
                                               ba.o_part, ba.lse_part, case["w_uv"], ba.out, ba.lse))

    def plan_lead(self, steps=5):
        """Times the calls alone (equal chunks) and picks the absorb plan's lead for the
        step: the absorb decode's CTAs on its short chunks leave their SMs to the GQA
        decode, those on the lead chunks keep the SMs it leaves idle busy."""
        self.call_ms = self.time_calls(steps)
        if not self.use_lead:
            return
        self.lead = self.gqla.gqla_plan_lead(
            self.dims, self.s_q, torch.cuda.get_device_properties(self.dev).multi_processor_count,
            self.splits["absorb"], self.splits["gqa"],
            self.call_ms["decode_absorb"] * 1e3, self.call_ms["decode_gqa"] * 1e3,
            self.call_ms["combine_absorb"] * 1e3)

    def step(self):
        # query absorption first, then the GQA path (one call) on its own stream beside
        # the absorb path's decode and combine; the step ends when both are done.  With a
        # lead in the absorb plan the absorb decode is launched first, so that its CTAs
        # are placed before the GQA decode's, which then take the SMs of the short chunks
        calls = self.calls
        gqa_step = self.gqa_step_call(self.case["q"], self.kv)
        main = torch.cuda.current_stream()
        calls[0]()
        fork = torch.cuda.Event()
        fork.record(main)
        self.gqa_stream.wait_event(fork)
        if self.lead[0] > 0:
            dec, comb = self.lead_calls(self.case["q"], self.kv, self.ba, self.lead)
            dec()
            with torch.cuda.stream(self.gqa_stream):
                gqa_step()
            comb()
        else:
            with torch.cuda.stream(self.gqa_stream):
                gqa_step()
            calls[1]()
            calls[2]()
        join = torch.cuda.Event()
        join.record(self.gqa_stream)
        main.wait_event(join)

    def capture(self, warmup):
        """The step as one CUDA graph (the launches replay without host overhead, each
        kernel's set-up overlapping the previous kernel's tail on its stream), and a
        second graph running the calls in order with an event record around each; the
        latter's times plan the step's absorb lead before the step is captured."""
        for _ in range(warmup):
            flush_l2(self.dev)
            self.step()
        torch.cuda.synchronize()
        self.gev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(self.calls) + 1)]
        self.graph_ev = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph_ev):
            for i, c in enumerate(self.calls):
                self.gev[i].record()
                c()
            self.gev[-1].record()
        # each path's step alone, as a user of that path runs it (its calls back to back on
        # one stream, each kernel's set-up overlapping its predecessor's tail)
        self.graph_path = {}
        for path, cs in (("absorb", self.calls[:3]), ("gqa", [self.gqa_step_call(self.case["q"], self.kv)])):
            g_ = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_):
                for c in cs:
                    c()
            self.graph_path[path] = g_
        for g_ in (self.graph_ev, *self.graph_path.values()):
            for _ in range(warmup):
                flush_l2(self.dev)
                g_.replay()
        torch.cuda.synchronize()
        self.plan_lead()
        for _ in range(warmup):
            flush_l2(self.dev)
            self.step()
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.step()
        for _ in range(warmup):
            flush_l2(self.dev)
            self.graph.replay()
        torch.cuda.synchronize()

    def time_steps(self, steps, graph=None):
        """Per-step device times (ms) of `steps` replays, issued back to back (an L2
        flush outside each step's event pair), one synchronize at the end."""
        graph = graph or self.graph
        stream = torch.cuda.current_stream()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for e0, e1 in ev:
            flush_l2(self.dev)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        return [e0.elapsed_time(e1) for e0, e1 in ev]

    def time_paths(self, steps):
        """Mean device time (ms) of each path's step graph."""
        return {path: sum(self.time_steps(steps, g_)) / steps for path, g_ in self.graph_path.items()}

    def time_calls(self, steps):
        per_call = [[] for _ in self.calls]
        for _ in range(steps):
            flush_l2(self.dev)
            self.graph_ev.replay()
            torch.cuda.synchronize()
            for i in range(len(self.calls)):
                per_call[i].append(self.gev[i].elapsed_time(self.gev[i + 1]))
        return {n: sum(v) / len(v) for n, v in zip(CALL_NAMES, per_call)}

    def check_device_errors(self):
        st_a, _ = self.gqla.gqla_read_device_error(self.ba.workspace)
        st_g, _ = self.gqla.gqla_read_device_error(self.bg.workspace)
        if st_a or st_g:
            raise RuntimeError(f"device-side error during the bench ({self.name}): {st_a} {st_g}")

    def e2e(self, steps, warmup, parts=None):
        """Host buffers through the C ABI, copies inside the timed region.  The batch is
        cut into `parts` sub-batches of whole sequences, each a complete step of its own
        (its own split plan and buffers), so that one part's host copies overlap another
        part's kernels: every input copy runs on a copy-in stream (q, then the page table
        and lengths as one int32 buffer, part by part), each part's query absorption and
        absorb path run on the main stream, its GQA path on a second stream, and each
        output goes back on a copy-out stream as soon as its path is done.  The step ends
        when every copy has landed.  Returns (ms, h2d, d2h, parts)."""
        gqla, dev, case = self.gqla, self.dev, self.case
        if parts is None:
            parts = [1, 1] if self.B >= 8 else [1]
        elif isinstance(parts, int):
            parts = [1] * parts
        weights = [float(x) for x in parts]
        pt_c, sl_c = case["page_table"].cpu(), case["seqlens"].cpu()
        q_h = case["q"].cpu().pin_memory()
        q_e = torch.empty_like(case["q"])
        outa_h = torch.empty(self.ba.out.shape, dtype=torch.bfloat16).pin_memory()
        outg_h = torch.empty(self.bg.out.shape, dtype=torch.bfloat16).pin_memory()
        h, s_q = self.w.num_heads, self.s_q
        # sub-batch boundaries in whole sequences, in proportion to the weights
        acc = [sum(weights[:k]) for k in range(len(weights) + 1)]
        cuts = [round(self.B * a / acc[-1]) for a in acc]
        if any(b1 <= b0 for b0, b1 in zip(cuts, cuts[1:])):
            raise ValueError(f"sub-batch weights {parts} leave an empty sub-batch of {self.B} sequences")
        lanes = []
        h2d = q_h.numel() * 2
        for k in range(len(weights)):
            b0, b1 = cuts[k], cuts[k + 1]
            pt_k, sl_k = pt_c[b0:b1].contiguous(), sl_c[b0:b1].contiguous()
            meta_h = torch.cat([pt_k.flatten(), sl_k]).pin_memory()
            meta_d = torch.empty(meta_h.shape, dtype=torch.int32, device=dev)
            kv = gqla.make_kv_index(meta_d[:pt_k.numel()].view(pt_k.shape), meta_d[pt_k.numel():],
                                    case["num_pages"])
            sa = gqla.plan_splits("absorb", h, s_q, sl_k)
            sg = gqla.plan_splits("gqa", h, s_q, sl_k, fused=True)
            ba = gqla.DecodeBuffers(self.dims, b1 - b0, s_q, sa, "absorb", device=dev)
            bg = gqla.DecodeBuffers(self.dims, b1 - b0, s_q, sg, "gqa", device=dev)
            q_k = q_e[b0:b1]
            # the sub-batch's absorb lead, from the whole batch's call times scaled to its
            # pages per chunk (only with --e2e-lead: the sub-batches overlap one another's
            # paths, which the lead's model does not cover)
            lead = (0, 16)
            if self.e2e_lead and self.lead[0] > 0 and self.call_ms:
                pg_all = int(((sl_c + gqla.PAGE_SIZE - 1) // gqla.PAGE_SIZE).sum())
                pg_k = int(((sl_k + gqla.PAGE_SIZE - 1) // gqla.PAGE_SIZE).sum())
                ta = self.call_ms["decode_absorb"] * 1e3 * (pg_k / sa) / (pg_all / self.splits["absorb"])
                tg = self.call_ms["decode_gqa"] * 1e3 * (pg_k / sg) / (pg_all / self.splits["gqa"])
                tc = self.call_ms["combine_absorb"] * 1e3 * pg_k / pg_all
                sms = torch.cuda.get_device_properties(dev).multi_processor_count
                lead = gqla.gqla_plan_lead(self.dims, s_q, sms, sa, sg, ta, tg, tc)
            if lead[0] > 0:
                dec_k, comb_k = self.lead_calls(q_k, kv, ba, lead)
            else:
                dec_k = lambda kv=kv, ba=ba: gqla.gqla_decode_absorb(self.dims, ba.q_absorbed, case["latent"], kv,
                                                                      ba.num_splits, ba.o_part, ba.lse_part, ba.workspace)
                comb_k = lambda kv=kv, ba=ba: gqla.gqla_combine(self.dims, kv, s_q, ba.num_splits, 512, ba.o_part,
                                                                 ba.lse_part, case["w_uv"], ba.out, ba.lse)
            lanes.append(dict(b0=b0, b1=b1, meta_h=meta_h, meta_d=meta_d, kv=kv, ba=ba, bg=bg, q=q_k, lead=lead,
                              absorb=[lambda q_k=q_k, ba=ba: gqla.gqla_absorb_query(self.dims, q_k, case["w_uk"], ba.q_absorbed),
                                      dec_k, comb_k],
                              gqa=lambda q_k=q_k, kv=kv, bg=bg: gqla.gqla_decode_gqa_step(
                                  self.dims, q_k, self.kvx, self.kr, kv, bg.num_splits, bg.o_part, bg.lse_part,
                                  bg.out, bg.lse, bg.workspace)))
            h2d += meta_h.numel() * 4
        d2h = outa_h.numel() * 2 + outg_h.numel() * 2
        copy_in, copy_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

        def e2e_step():
            main = torch.cuda.current_stream()
            begin = torch.cuda.Event()
            begin.record(main)
            copy_in.wait_event(begin)
            copy_out.wait_event(begin)
            arrived = []
            with torch.cuda.stream(copy_in):
                for ln in lanes:
                    ln["q"].copy_(q_h[ln["b0"]:ln["b1"]], non_blocking=True)
                    ln["meta_d"].copy_(ln["meta_h"], non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(copy_in)
                    arrived.append(ev)
            for ln, ev in zip(lanes, arrived):
                main.wait_event(ev)
                self.gqa_stream.wait_event(ev)
                if ln["lead"][0] > 0:  # the absorb decode first (see step())
                    ln["absorb"][0]()
                    ln["absorb"][1]()
                with torch.cuda.stream(self.gqa_stream):
                    ln["gqa"]()
                gqa_done = torch.cuda.Event()
                gqa_done.record(self.gqa_stream)
                for c in (ln["absorb"][2:] if ln["lead"][0] > 0 else ln["absorb"]):
                    c()
                absorb_done = torch.cuda.Event()
                absorb_done.record(main)
                with torch.cuda.stream(copy_out):
                    copy_out.wait_event(gqa_done)
                    outg_h[ln["b0"]:ln["b1"]].copy_(ln["bg"].out, non_blocking=True)
                    copy_out.wait_event(absorb_done)
                    outa_h[ln["b0"]:ln["b1"]].copy_(ln["ba"].out, non_blocking=True)
            done = torch.cuda.Event()
            done.record(copy_out)
            main.wait_event(done)
            gqa_end = torch.cuda.Event()
            gqa_end.record(self.gqa_stream)
            main.wait_event(gqa_end)

        for _ in range(warmup):  # eager warm-up, then the same step as one graph
            e2e_step()
        torch.cuda.synchronize()
        graph_e2e = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_e2e):
            e2e_step()
        for _ in range(warmup):
            graph_e2e.replay()
        torch.cuda.synchronize()
        times = self.time_steps(steps, graph_e2e)
        for i, ln in enumerate(lanes):
            for name, host, dev_out in (("absorb", outa_h, ln["ba"].out), ("gqa", outg_h, ln["bg"].out)):
                got, ref = host[ln["b0"]:ln["b1"]], dev_out.cpu()
                if not torch.equal(got, ref):
                    bad = (got != ref)
                    raise RuntimeError(
                        f"end-to-end outputs differ from the device results: sub-batch {i} "
                        f"({ln['b0']}..{ln['b1']}), {name} path, {int(bad.sum())} of {bad.numel()} values, "
                        f"first at {tuple(int(x) for x in bad.nonzero()[0])}, NaN in copy "
                        f"{int(torch.isnan(got.float()).sum())} / on device {int(torch.isnan(ref.float()).sum())}")
        # the sub-batches' results agree with the whole batch's (other split plans: fp32
        # merges in another order, so within rounding, not bit for bit)
        for got, ref in ((outa_h, self.ba.out), (outg_h, self.bg.out)):
            diff = (got.float() - ref.float().cpu()).abs().max().item()
            if not diff <= 2e-2:
                raise RuntimeError(f"sub-batched outputs differ from the whole batch's by {diff}")
        self.e2e_leads = [list(ln["lead"]) for ln in lanes]
        return sum(times) / len(times), h2d, d2h, [b1 - b0 for b0, b1 in zip(cuts, cuts[1:])]

    def report(self, mean, world, path_ms=None):
        """Per-kernel and per-path roofline fractions from the per-call means (ms)."""
        acc, counts = accounting(self.w, self.case, self.s_q, self.splits["gqa"])
        acc_a, _ = accounting(self.w, self.case, self.s_q, self.splits["absorb"])
        acc["decode_absorb"] = acc_a["decode_absorb"]
        acc["combine_absorb"] = acc_a["combine_absorb"]
        peaks, peak_kind = _peaks()
        hbm_peak = float(peaks["hbm_gbs"])
        tc_peak = float(peaks["bf16_tflops"])
        tokens_step = self.B * self.s_q

        def roof(name):
            sec = mean[name] * 1e-3
            gbs = acc[name]["bytes"] / sec / 1e9
            tfs = acc[name]["flops"] / sec / 1e12
            return {"us": mean[name] * 1e3, "hbm_gbs": gbs, "hbm_frac": gbs / hbm_peak,
                    "tflops": tfs, "tensor_frac": tfs / tc_peak}

        per_kernel = {n: roof(n) for n in CALL_NAMES}
        total = sum(mean.values())
        for n in CALL_NAMES:
            per_kernel[n]["share"] = mean[n] / total
        dominant = max(CALL_NAMES, key=lambda n: mean[n])
        dk = per_kernel[dominant]
        t_mem = acc[dominant]["bytes"] / (hbm_peak * 1e9)
        t_cmp = acc[dominant]["flops"] / (tc_peak * 1e12)
        if t_cmp > t_mem:
            roofline = {"bound": "tensor", "achieved": dk["tflops"], "peak": tc_peak,
                        "unit": "TFLOP/s", "frac": dk["tensor_frac"]}
        else:
            roofline = {"bound": "hbm", "achieved": dk["hbm_gbs"], "peak": hbm_peak,
                        "unit": "GB/s", "frac": dk["hbm_frac"]}
        roofline.update({"kernel": dominant,
                         "peak_source": (f"{peak_kind} (MEASURED_PEAKS.json burst)"
                                         if peak_kind == "measured" else "fallback"),
                         "algorithmic_bytes_per_launch": acc[dominant]["bytes"],
                         "algorithmic_flops_per_launch": acc[dominant]["flops"],
                         "traffic": _stored_traffic(dominant, self.name, self.s_q)})

        def path_info(kernels, dec, path):
            # the path's own step graph when timed, else its calls' event-separated times
            us = (path_ms[path] if path_ms else sum(mean[k] for k in kernels)) * 1e3
            t_m = acc[dec]["bytes"] / (hbm_peak * 1e9)
            t_c = acc[dec]["flops"] / (tc_peak * 1e12)
            bound = "tensor" if t_c > t_m else "hbm"
            frac = (t_c if bound == "tensor" else t_m) / (mean[dec] * 1e-3)
            return {"us_per_step": us, "tokens_per_s": world * tokens_step / (us * 1e-6),
                    "decode_kernel": dec, "decode_us": mean[dec] * 1e3, "binding": bound,
                    "binding_roofline_frac": frac, "hbm_frac": per_kernel[dec]["hbm_frac"],
                    "tensor_frac": per_kernel[dec]["tensor_frac"]}

        per_path = {"absorb": path_info(["absorb_query", "decode_absorb", "combine_absorb"], "decode_absorb", "absorb"),
                    "gqa": path_info(["decode_gqa", "combine_gqa"], "decode_gqa", "gqa")}
        return roofline, per_path, per_kernel, acc

    def config(self, world):
        w = self.w
        return {"workload": self.name, "num_heads": w.num_heads, "num_groups": w.num_groups,
                "batch": self.B,
                "context": w.lengths[1] if w.lengths[0] == "fixed" else list(w.lengths[1:]),
                "s_q": self.s_q, "paged": w.paged, "paths": ["absorb", "gqa"],
                "tokens_per_step": self.B * self.s_q, "num_splits": self.splits,
                "absorb_lead": list(self.lead),
                "l2": "flushed (256 MiB write + 256 MiB read) before every timed step",
                "parallelism": f"replicas x{world} (independent batches per GPU)"}


def measure_other_workloads(args, headline, dev):
    """Every other workload (and s_q) of the suite on this GPU: step time, per-call
    times and each path's roofline fractions (no end-to-end leg, no CPU baseline)."""
    from decode_attention_06_b200 import synth
    out = {}
    for name, w in synth.WORKLOADS.items():
        for s in w.s_q:
            if (name, s) == headline:
                continue
            wb = Workbench(name, s, 0, dev, args.splits, lead=not args.no_lead)
            wb.time_expand()
            wb.capture(args.warmup)
            ms = wb.time_steps(args.steps)
            mean = wb.time_calls(args.steps)
            path_ms = wb.time_paths(args.steps)
            wb.check_device_errors()
            _, per_path, per_kernel, _ = wb.report(mean, 1, path_ms)
            out[f"{name}/sq{s}"] = {
                "ms_per_step": sum(ms) / len(ms),
                "tokens_per_s": wb.B * s / (sum(ms) / len(ms) * 1e-3),
                "num_splits": wb.splits, "absorb_lead": list(wb.lead), "per_path": per_path,
                "per_kernel_us": {n: per_kernel[n]["us"] for n in CALL_NAMES}}
            del wb
            torch.cuda.empty_cache()
    return out


def run_tp(args, rank, world, dev):
    """Group-axis tensor parallelism of the GQA path over the `world` ranks (strong
    scaling: every rank holds g / world groups of the same batch's expanded cache and
    decodes its h / world heads; an in-place NCCL all-gather assembles the heads).
    Each step = the rank's decode + combine + the gather, timed on the device, max
    over ranks."""
    from decode_attention_06_b200 import gqla, synth
    from decode_attention_06_b200.tp import GqaTensorParallel, GroupShard
    w = synth.WORKLOADS[args.workload]
    s_q = args.s_q or w.s_q[0]
    if w.num_groups % world:
        return {"skipped": f"{w.num_groups} groups do not split over {world} ranks"}
    case = synth.make_case(w.num_heads, w.num_groups, w.seqlens(), s_q, paged=w.paged,
                           seed=w.seed, device=str(dev))  # the same batch on every rank
    shard = GroupShard(w.num_heads, w.num_groups, rank, world)
    B = case["seqlens"].numel()
    n_slots = case["num_pages"] * case["page_size"]
    kv = gqla.make_kv_index(case["page_table"], case["seqlens"], case["num_pages"])
    splits = args.splits or gqla.plan_splits("gqa", shard.heads, s_q, case["seqlens"].cpu())
    tp = GqaTensorParallel(shard, B, s_q, splits, dev)
    kvx = torch.empty(shard.groups, n_slots, 256, dtype=torch.bfloat16, device=dev)
    kr = torch.empty(n_slots, 64, dtype=torch.bfloat16, device=dev)
    gqla.gqla_expand_cache(tp.dims, case["latent"], shard.slice_groups(case["w_uk"]),
                           shard.slice_groups(case["w_uv"]), kvx, kr)
    q_local = shard.slice_heads(case["q"])
    del case
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        flush_l2(dev)
        tp.step(q_local, kvx, kr, kv)
    torch.cuda.synchronize()
    torch.distributed.barrier()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for e0, e1, e2 in ev:
        flush_l2(dev)
        e0.record(stream)
        tp.local_step(q_local, kvx, kr, kv)
        e1.record(stream)
        tp.gather()
        e2.record(stream)
    torch.cuda.synchronize()
    st, _ = gqla.gqla_read_device_error(tp.bufs.workspace)
    if st:
        raise RuntimeError(f"device-side error in the tensor-parallel step: {st}")
    t = torch.tensor([sum(e0.elapsed_time(e2) for e0, _, e2 in ev) / args.steps,
                      sum(e0.elapsed_time(e1) for e0, e1, _ in ev) / args.steps],
                     dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    ms, local_ms = float(t[0]), float(t[1])
    return {"scaling": "strong", "ranks": world, "groups_per_rank": shard.groups,
            "heads_per_rank": shard.heads, "num_splits": splits, "ms_per_step": ms,
            "local_decode_combine_ms": local_ms, "tokens_per_s": B * s_q / (ms * 1e-3),
            "gather_bytes_per_rank": tp.out_all.numel() * 2 + tp.lse_all.numel() * 4,
            "note": "each rank: gqla_decode_gqa + gqla_combine on its groups, then an in-place "
                    "NCCL all-gather of the heads; device time, max over ranks"}


def run_ours(args, rank, world, local_rank):
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wb = Workbench(args.workload, args.s_q, rank, dev, args.splits, lead=not args.no_lead)
    wb.e2e_lead = args.e2e_lead
    expand_ms, expand_tc_ms = wb.time_expand()
    wb.capture(args.warmup)

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        step_ms = wb.time_steps(args.steps)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ms_step = sum(step_ms) / args.steps
    mean = wb.time_calls(args.steps)
    path_ms = wb.time_paths(args.steps)
    wb.check_device_errors()
    e2e_arg = None
    if args.e2e_parts:
        e2e_arg = [float(x) for x in args.e2e_parts.split(",")] if "," in args.e2e_parts else int(args.e2e_parts)
    e2e_ms, h2d, d2h, e2e_parts = wb.e2e(args.steps, args.warmup, e2e_arg)

    # ---- max over ranks
    tokens_step = wb.B * wb.s_q
    ms_step, e2e_ms, value, e2e_value = aggregate_over_ranks(ms_step, e2e_ms, world, tokens_step, dev)
    roofline, per_path, per_kernel, acc = wb.report(mean, world, path_ms)
    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 cache/queries, N(0,1/512) bf16 W_UK/W_UV)",
        "config": wb.config(world),
        "roofline": roofline,
        "per_path": per_path,
        "per_kernel": per_kernel,
        "expand": {"ms": expand_ms, "slots": wb.n_slots,
                   "tflops": acc["expand"]["flops"] / (expand_ms * 1e-3) / 1e12,
                   "tc_ms": expand_tc_ms,
                   "tc_tflops": acc["expand"]["flops"] / (expand_tc_ms * 1e-3) / 1e12},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "sub_batches": e2e_parts,
                "absorb_leads": wb.e2e_leads},
        "gpu_launches": wb.launches_per_step() * args.steps,
        "clocks": clocks.summary(),
    }
    if args.sparse_topk:
        result["sparse"] = run_sparse(args, wb.dims, wb.case, wb.s_q, wb.kvx, wb.kr, wb.kv,
                                      lambda: flush_l2(dev), float(_peaks()[0]["hbm_gbs"]))
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, cores, what = cpu_oracle_rate(wb.case, wb.w, wb.s_q, budget_s=args.cpu_budget)
        result["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": cores,
                                  "kind": "oracle", "sample": what}
    if world == 1 and not args.headline_only:
        headline = (wb.name, wb.s_q)
        del wb
        torch.cuda.empty_cache()
        result["workloads"] = measure_other_workloads(args, headline, dev)
    if world > 1:
        del wb
        torch.cuda.empty_cache()
        result["tp"] = run_tp(args, rank, world, dev)
    return result


def run_sparse(args, dims, case, s_q, kvx, kr, kv, flush_l2, hbm_peak):
    """Sparse GQLA on the GQA path: every query token attends to --sparse-topk
    seeded positions of its visible context.  Two forms, each timed like the step
    (one graph, L2 flushed before each replay) and per call: the selected cache
    (gather the rows, GQA decode over them, combine) and the fused one (slot lists,
    the GQA decode gathering the rows itself with tile::gather4, combine)."""
    from decode_attention_06_b200 import gqla, synth
    B = case["seqlens"].numel()
    topk = args.sparse_topk
    idx = synth.make_topk(case["seqlens"].cpu(), s_q, topk, seed=77).to(case["q"].device)
    splits = args.splits or gqla.gqla_num_splits_hint("gqa", dims.num_heads, 1)
    n_slots = kv.num_pages * kv.page_size
    tok_bytes = 2 * (2 * dims.num_groups * 128 + 64)
    q_bytes = B * s_q * dims.num_heads * 192 * 2

    def measure(fused):
        sb = gqla.SparseBuffers(dims, B, s_q, topk, splits, device=case["q"].device, fused=fused)
        if fused:
            names = ["select", "decode_gqa_sparse", "combine"]
            calls = [
                lambda: gqla.gqla_sparse_select(dims, kv, s_q, idx, sb.sel_slot, sb.sel_page_table,
                                                sb.sel_seqlens, sb.workspace),
                lambda: gqla.gqla_decode_gqa_sparse(dims, case["q"], kvx, kr, n_slots, sb.sel_index, sb.sel_slot,
                                                    splits, sb.dec.o_part, sb.dec.lse_part, sb.workspace)]
        else:
            names = ["gather", "decode_gqa", "combine"]
            q1 = case["q"].view(B * s_q, 1, dims.num_heads, 192)
            calls = [
                lambda: gqla.gqla_sparse_gather(dims, kvx, kr, kv, s_q, idx, sb.kv_sel, sb.k_rope_sel,
                                                sb.sel_page_table, sb.sel_seqlens, sb.workspace),
                lambda: gqla.gqla_decode_gqa(dims, q1, sb.kv_sel, sb.k_rope_sel, sb.sel_index, splits,
                                             sb.dec.o_part, sb.dec.lse_part, sb.workspace)]
        calls.append(lambda: gqla.gqla_combine(dims, sb.sel_index, 1, splits, 128, sb.dec.o_part,
                                               sb.dec.lse_part, None, sb.dec.out, sb.dec.lse))
        ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(calls) + 1)]

        def step(events=None):
            for i, c in enumerate(calls):
                if events is not None:
                    events[i].record()
                c()
            if events is not None:
                events[-1].record()

        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        graphs = []
        for events in (None, ev):
            g_ = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_):
                step(events)
            graphs.append(g_)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t_step, t_call = [], [[] for _ in calls]
        for _ in range(args.steps):
            flush_l2()
            e0.record()
            graphs[0].replay()
            e1.record()
            torch.cuda.synchronize()
            t_step.append(e0.elapsed_time(e1))
            flush_l2()
            graphs[1].replay()
            torch.cuda.synchronize()
            for i in range(len(calls)):
                t_call[i].append(ev[i].elapsed_time(ev[i + 1]))
        st, _ = gqla.gqla_read_device_error(sb.workspace)
        if st:
            raise RuntimeError(f"device-side error in the sparse step: {st}")
        n_sel = int(sb.sel_seqlens.sum())
        ms = sum(t_step) / len(t_step)
        us = {n: 1e3 * sum(v) / len(v) for n, v in zip(names, t_call)}
        # one pass over the selected rows, the queries and the output: what a single
        # kernel would have to move at least
        fused_bytes = n_sel * tok_bytes + q_bytes + B * s_q * dims.num_heads * 128 * 2
        return {"us_per_step": ms * 1e3, "tokens_per_s": B * s_q / (ms * 1e-3), "per_call_us": us,
                "selected_tokens": n_sel, "min_bytes": fused_bytes,
                "hbm_frac_of_min_bytes": fused_bytes / (ms * 1e-3) / 1e9 / hbm_peak}

    return {"topk": topk, "selected_cache": measure(False), "fused": measure(True),
            "selection": "seeded uniform distinct visible positions (synth.make_topk)"}


def run_reference(args, rank, world):
    """The oracle as the reference arm: each step decodes one (sequence, group)
    unit of the workload on the host cores."""
    from decode_attention_06_b200 import synth
    import oracle
    w = synth.WORKLOADS[args.workload]
    s_q = args.s_q or w.s_q[0]
    case = synth.make_case(w.num_heads, w.num_groups, w.seqlens(), s_q, paged=w.paged,
                           seed=w.seed)
    B = case["seqlens"].numel()
    times = []
    for k in range(args.warmup + args.steps):
        b = k % B
        q, lat, pt, sl = _gather(case, [b])
        t0 = time.perf_counter()
        oracle.decode(q, lat, pt, sl, case["w_uk"], case["w_uv"], w.num_groups,
                      units=[(0, k % w.num_groups)])
        if k >= args.warmup:
            times.append(time.perf_counter() - t0)
    ms = 1e3 * sum(times) / len(times)
    tokens = s_q / w.num_groups  # one group of one sequence = 1/g of its s_q tokens
    value = tokens / (ms * 1e-3)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same generator and workload as the GPU arm)",
        "config": {"workload": args.workload, "num_heads": w.num_heads,
                   "num_groups": w.num_groups, "batch": B, "s_q": s_q,
                   "paths": ["un-absorbed definition"]},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": "one (sequence, group) unit per step: all heads of one "
                                   "group of one sequence, fp64"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def ncu_summary(csv_path):
    """Per-kernel launch count, total and share of device time from an ncu
    `--metrics gpu__time_duration.sum --csv` launch list (host-side only)."""
    import collections
    import csv
    rows = [r for r in csv.reader(open(csv_path)) if len(r) > 5]
    idx = {h: i for i, h in enumerate(rows[0])}
    agg = collections.defaultdict(lambda: [0, 0.0])
    for r in rows[1:]:
        if r[idx["Metric Name"]] != "gpu__time_duration.sum":
            continue
        name = r[idx["Kernel Name"]].split("(")[0].replace("void ", "")
        for junk in ("(anonymous namespace)::", "<unnamed>::", "unnamed>::"):
            name = name.replace(junk, "")
        scale = {"ns": 1e-3, "us": 1.0, "usecond": 1.0, "nsecond": 1e-3, "ms": 1e3,
                 "msecond": 1e3}.get(r[idx["Metric Unit"]], 1.0)
        agg[name[:80]][0] += 1
        agg[name[:80]][1] += float(r[idx["Metric Value"]].replace(",", "")) * scale
    total = sum(v[1] for v in agg.values())
    print(f"{'launches':>8} {'total us':>11} {'share':>7}  kernel")
    for k, (n, t) in sorted(agg.items(), key=lambda x: -x[1][1]):
        print(f"{n:8d} {t:11.1f} {100 * t / total:6.1f}%  {k}")


def aggregate_over_ranks(ms_step, e2e_ms, world, tokens_per_rank, device):
    """Replicas: every rank decodes its own batch.  The job's step time is the
    slowest rank's (max over ranks); its throughput counts every rank's tokens."""
    t = torch.tensor([ms_step, e2e_ms], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    ms_step, e2e_ms = float(t[0]), float(t[1])
    value = world * tokens_per_rank / (ms_step * 1e-3)
    e2e_value = world * tokens_per_rank / (e2e_ms * 1e-3)
    return ms_step, e2e_ms, value, e2e_value


def _relaunch_under_torchrun(n):
    """`bench.py --gpus N` (N > 1) started outside torchrun: run the same command as
    N ranks, one process per GPU, and pass on their exit status."""
    import socket
    import subprocess
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__),
           *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--s-q", dest="s_q", type=int, default=None)
    ap.add_argument("--splits", type=int, default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--headline-only", action="store_true",
                    help="measure the headline workload only (not the rest of the suite)")
    ap.add_argument("--sparse-topk", type=int, default=0,
                    help="also time sparse GQLA with this many selected positions per query token")
    ap.add_argument("--e2e-parts", default=None,
                    help="sub-batches of the end-to-end step: a count (equal parts) or relative "
                         "sizes such as 1,2,1 (default two equal parts from 8 sequences up, else 1)")
    ap.add_argument("--e2e-lead", action="store_true",
                    help="give the end-to-end sub-batches absorb leads too (scaled from the step's)")
    ap.add_argument("--no-lead", action="store_true",
                    help="equal absorb chunks in the step too (no lead planned beside the GQA path)")
    ap.add_argument("--ncu-summary", metavar="CSV", default=None,
                    help="print the per-kernel summary of an ncu launch list and exit")
    args = ap.parse_args()
    if args.ncu_summary:
        ncu_summary(args.ncu_summary)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")

    env_world = os.environ.get("WORLD_SIZE")
    if env_world is None and args.gpus > 1 and args.impl == "ours":
        sys.exit(_relaunch_under_torchrun(args.gpus))
    world = int(env_world or "1")
    if args.impl == "ours" and world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE is {world}: launch one rank per GPU")
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
