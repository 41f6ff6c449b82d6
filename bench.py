"""Benchmark: OmniKVQuant decode step (cache append + fused split-K decode +
combine/inverse rotation, every layer) on synthetic inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl omnikv|reference] [--workload omni30b-b8]
    torchrun --nproc-per-node N bench.py --gpus N ...   (one rank per GPU, weak scaling)

Default workload: the largest single-GPU configuration, the Qwen3-Omni-30B-A3B-
shaped decode (48 layers, 32 query / 4 KV heads, head dim 128, batch 8, 65,536
cached tokens per sequence in an audio-heavy interleaved layout, K2/V2, 32-token
windows); one step appends one text token per sequence to every layer's cache
and runs decode attention for every layer. Each rank runs its own batch
(different seed), so per-GPU work is fixed as N grows.

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events on
the launching stream and preceded by an untimed L2 flush (a 512 MiB write);
barrier + synchronize around the timed region; the max over ranks is reported.
All steps are replayed from one CUDA graph holding, per step, the L2 flush, the
step's start event, exactly the C-ABI calls of the step, and its end event (no
host gaps between steps). `value` has all inputs resident in HBM; `e2e` also
copies each step's inputs (q, k, v and modality ids of every layer, packed per
layer in pinned host memory) and the step's outputs back to the host, inside the
step's timed region, on side streams (layer 0's inputs first, the other layers'
while layer 0 decodes; all outputs but the last layer's while it decodes), captured
the same way.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

if "reference" in sys.argv:  # the oracle arm: one thread per BLAS / OpenMP pool from the start
    for _var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ.setdefault(_var, "1")

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS_KEYS = ("tiny", "omni3b-b1", "omni3b-b16", "omni30b-b8", "ragged-b64")

METRIC = "2-bit decode attention tokens/s and achieved HBM GB/s vs ~8 TB/s (1 B200)"
UNIT = "tokens/s"
# algorithmic packed bytes per token per kv head: (key bits, value bits, key metadata format)
BYTES_PER_TOKEN_HEAD = {(2, 2, "fp16"): 82, (4, 4, "fp16"): 146, (2, 2, "mx"): 70.5, (4, 4, "mx"): 134.5,
                        (2, 2, "turbo"): 68, (4, 4, "turbo"): 132}
META_FORMATS = {"fp16": 0, "mx": 1, "turbo": 2}   # omnikv_config.key_meta_format

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the
# timed kernel, per (workload, key metadata format), from an ncu capture of this
# benchmark (its summary is kept with the other profiles), valid for the kernel
# sources with this SHA-256; any change to them makes the field null until the
# next capture.
TRAFFIC_CAPTURES = {
    ("qwen3-omni-30b-48L-b8-ctx65536", "fp16"): {
        "sources_sha256": "e667514f81980f6b28074c51c3f79cb8d4094517921d6e109946c792ce697e40",
        "bytes_per_launch": 173712384 + 8849664},
}
KERNEL_SOURCES = ("decode_split_k.cu", "decode_common.cuh", "append.cuh", "common.cuh", "ptx.cuh", "kernels.h")


def kernel_sources_sha256():
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(os.path.dirname(os.path.abspath(__file__)), "bit_kv_cache_pack_b200", "csrc")
    for name in KERNEL_SOURCES:
        with open(os.path.join(d, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def captured_traffic(workload_name, meta="fp16"):
    cap = TRAFFIC_CAPTURES.get((workload_name, meta))
    if cap is None:
        return None
    return cap["bytes_per_launch"] if kernel_sources_sha256() == cap["sources_sha256"] else None


L2_FLUSH_BYTES = 512 << 20


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=4)
    ap.add_argument("--impl", default="omnikv", choices=["omnikv", "reference"])
    ap.add_argument("--workload", default="omni30b-b8", choices=sorted(WORKLOADS_KEYS))
    ap.add_argument("--no-graphs", action="store_true")
    ap.add_argument("--layer", choices=["decode", "write", "calibrate"], default=None,
                    help="time one layer's decode (+ combine) or prefill cache write on --workload instead of "
                         "the decode step (one JSON line per split count), or the value-basis calibration of one "
                         "(layer, kv head) from the workload's first sequence")
    ap.add_argument("--bits", type=int, default=0, help="with --layer: 2 or 4 (default: the workload's)")
    ap.add_argument("--meta", default="fp16", choices=sorted(META_FORMATS),
                    help="key metadata format: fp16 (m, s) pairs, mx (MXFP4, the pages' default) or turbo "
                         "(the TurboQuant key codec the pages compare against: one scale per token)")
    ap.add_argument("--batch", type=int, default=0, help="with --layer: override the workload's batch")
    ap.add_argument("--splits", default="0", help="with --layer decode: comma-separated split counts (0: default)")
    ap.add_argument("--stream", action="store_true",
                    help="with --layer decode: also time the streaming/captioning policy's decode "
                         "(packed body + tail + combine, omnikv_stream_decode) over the same cache")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clocks-csv", default=None, help="where to keep the nvidia-smi samples (default: a temp file)")
    return ap.parse_args()


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_seed(workload: str, rank: int) -> int:
    """Each rank decodes its own batch (weak scaling): a different seed per rank."""
    return WORKLOADS_KEYS.index(workload) + 1000 * rank


def workload_config(spec, world, meta="fp16"):
    """The `config` object of both arms' JSON lines: the workload and how it is
    measured (the same dict for the GPU arm and the oracle arm)."""
    from synth.workloads import seq_lengths
    L = seq_lengths(spec, 0)
    return {"workload": spec.name, "layers": spec.layers, "global_batch": spec.batch * world,
            "context": int(L.max()) if not spec.ragged else "%d..%d" % spec.ragged,
            "num_q_heads": spec.num_q_heads, "num_kv_heads": spec.num_kv_heads, "head_dim": 128,
            "key_bits": spec.key_bits, "value_bits": spec.value_bits, "window": 32,
            "key_meta_format": {"fp16": "fp16", "mx": "mxfp4", "turbo": "turbo (per-token key scale)"}[meta],
            "parallelism": "dp%d (independent sequences per rank)" % world,
            "l2": "GPU arm: flushed between timed steps (512 MiB write)"}


def max_over_ranks(values, device, world):
    """Elementwise maximum over all ranks of a list of timings (ms)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, path=None):
        import tempfile
        self.idx = gpu_index
        self.proc = None
        self.path = path or os.path.join(tempfile.gettempdir(), "omnikv_clocks_%d_%d.csv" % (os.getpid(), gpu_index))

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        return self.parse(self.path)

    @staticmethod
    def parse(path):
        """Median SM clock, the maximum, and the throttle reasons seen active in an
        nvidia-smi CSV of the query Q (None without samples)."""
        sm, smax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            for n, v in zip(names, parts[5:9]):  # a reason counts even where a clock is unreadable
                if v.lower() == "active":
                    reasons.add(n)
            try:
                sm.append(float(parts[1]))
                smax = max(smax, float(parts[2]))
            except ValueError:
                continue
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------
# the GPU arm
# ----------------------------------------------------------------------------
class Workload:
    """Per-layer constants and caches, prefilled (untimed), plus every step's inputs."""

    def __init__(self, spec, seed, device, total_steps, meta="fp16"):
        import bit_kv_cache_pack_b200 as m
        from synth.workloads import (codebook, decode_inputs, key_drift, layer_params, prefill_inputs,
                                     seq_lengths)
        self.m, self.spec, self.dev, self.meta = m, spec, device, meta
        self.lengths = seq_lengths(spec, seed)
        self.cap = int(-(-(int(self.lengths.max()) + total_steps) // 32) * 32)
        kb, vb = codebook(spec.key_bits), codebook(spec.value_bits)
        self.consts, self.caches = [], []
        qs, ks, vs, ms = [], [], [], []
        for layer in range(spec.layers):
            params = layer_params(spec, seed, layer)
            c = m.LayerConstants(kb, vb, params["key_signs"], params["value_rot"], spec.num_q_heads, device,
                                 key_meta_format=META_FORMATS[meta])
            cache = m.KVCache(spec.batch, spec.num_kv_heads, self.cap, spec.key_bits, spec.value_bits, device,
                              key_meta_format=META_FORMATS[meta])
            drift = key_drift(spec, seed, layer, self.cap // 32, device)
            if spec.ragged:
                for b in range(spec.batch):
                    k, v, mod = prefill_inputs(spec, seed, layer, params, drift, self.lengths, device,
                                               batch_index=[b])
                    n = int(self.lengths[b])
                    view = cache.sequence_view(b)
                    m.omnikv_write_cache(c.struct, view, k[:, :, :n].contiguous(), v[:, :, :n].contiguous(),
                                         mod[:, :n].contiguous(), n)
                    del k, v, mod
                cache.struct.max_seq_len = int(self.lengths.max())
            else:
                k, v, mod = prefill_inputs(spec, seed, layer, params, drift, self.lengths, device)
                m.omnikv_write_cache(c.struct, cache.struct, k, v, mod, int(self.lengths[0]))
                del k, v, mod
            torch.cuda.synchronize(device)
            self.consts.append(c)
            self.caches.append(cache)
            lq, lk, lv, lm = [], [], [], []
            for s in range(total_steps):
                q, kn, vn, mn = decode_inputs(spec, seed, layer, s, params, drift, self.lengths + s, device)
                lq.append(q), lk.append(kn), lv.append(vn), lm.append(mn)
            qs.append(torch.stack(lq)), ks.append(torch.stack(lk)), vs.append(torch.stack(lv))
            ms.append(torch.stack(lm))
        # [steps][layers][...] contiguous, so one step's inputs are one block
        self.q = torch.stack(qs, 1).contiguous()
        self.k = torch.stack(ks, 1).contiguous()
        self.v = torch.stack(vs, 1).contiguous()
        self.mod = torch.stack(ms, 1).contiguous()
        self.S, self.fused = m.omnikv_step_splits(self.consts[0].struct, self.caches[0].struct, 0)
        # the step's default split count grows (slightly) with the context: size
        # the partials for its value at the longest context of the run
        c0 = self.caches[0].struct
        saved = c0.max_seq_len
        c0.max_seq_len = int(self.lengths.max()) + total_steps - 1
        s_max = max(self.S, m.omnikv_step_splits(self.consts[0].struct, c0, 0)[0])
        c0.max_seq_len = saved
        self.part = m.partials_tensor(spec.batch, spec.num_q_heads, s_max, device)
        self.out = torch.empty(spec.layers, spec.batch, spec.num_q_heads, 128, dtype=torch.float32,
                               device=device)

    def step_calls(self, s, q, k, v, mod, stream, dec_events=None, before=None, after=None):
        """The C-ABI calls of one decode step over all layers: omnikv_decode_step
        per layer (the append-and-decode launch, then the combine launch). With
        `dec_events` (a start/end pair), layer s % layers makes the same step as
        its two calls, omnikv_append_decode between the events, so the dominant
        kernel (decode_step_kernel) is timed in place once per step. `before` and
        `after` (called with the layer index) let the end-to-end run order each
        layer after its input copy and its output copy after it."""
        m = self.m
        n = self.spec.layers
        for layer in range(n):
            if before is not None:
                before(layer)
            c, cache = self.consts[layer].struct, self.caches[layer].struct
            if dec_events is not None and layer == s % n:
                dec_events[0].record(stream)
                m.omnikv_append_decode(c, cache, q[layer], k[layer], v[layer], mod[layer], self.part, 0, stream)
                dec_events[1].record(stream)
                m.omnikv_combine_step(c, cache, self.part, 0, self.out[layer], stream)
            else:
                m.omnikv_decode_step(c, cache, q[layer], k[layer], v[layer], mod[layer], self.part, 0,
                                     self.out[layer], stream)
            if after is not None:
                after(layer)

    def launches_per_step(self, instrumented):
        """Library kernel launches in one step: 2 per layer (the append-and-decode
        launch and the combine launch) when the step's grid is resident at once,
        else 4 (append, decode, combine; the append is one launch for a token)."""
        return (2 if self.fused else 3) * self.spec.layers

    def decode_bytes(self, s):
        """Algorithmic bytes of one append-and-decode launch at step s (one
        layer): the packed records of every cached token and kv head after the
        append, 1 modality id per token, and the append itself per kv head (the
        new fp16 key and value read, the raw keys of the partial window read from
        the tail, the window record written)."""
        sp = self.spec
        L = self.lengths.astype(np.int64) + s
        T = (L + 1).sum()
        per_token = BYTES_PER_TOKEN_HEAD[(sp.key_bits, sp.value_bits, self.meta)]
        rec = int(per_token * 32)
        append = sp.num_kv_heads * int((512 + 256 * (L % 32) + rec).sum())
        return int(T * sp.num_kv_heads * per_token + T + append)


def run_gpu(args):
    import torch.distributed as dist
    from synth.workloads import WORKLOADS
    world, rank, local = dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    spec = WORKLOADS[args.workload]
    seed = rank_seed(args.workload, rank)
    K, W = args.steps, args.warmup
    total = W + K + K + 1  # device-resident run, then the e2e run
    wl = Workload(spec, seed, dev, total, args.meta)
    stream = torch.cuda.Stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    torch.cuda.synchronize(dev)

    # --- device-resident steps: one graph holding, per step, the L2 flush, the
    # start event, the step's C-ABI calls and the end event (no host gaps) -------
    ev = lambda: torch.cuda.Event(enable_timing=True, external=True)
    dec_ev = [(ev(), ev()) for _ in range(W + K)]
    step_ev = [(ev(), ev()) for _ in range(W + K)]
    use_graphs = not args.no_graphs
    graph = None
    if use_graphs:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            cs = torch.cuda.current_stream()
            for s in range(W + K):
                flush.zero_()
                step_ev[s][0].record(cs)
                wl.step_calls(s, wl.q[s], wl.k[s], wl.v[s], wl.mod[s], cs, dec_ev[s])
                step_ev[s][1].record(cs)
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local, args.clocks_csv)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    with torch.cuda.stream(stream):
        if use_graphs:
            graph.replay()
        else:
            for s in range(W + K):
                flush.zero_()
                step_ev[s][0].record(stream)
                wl.step_calls(s, wl.q[s], wl.k[s], wl.v[s], wl.mod[s], stream, dec_ev[s])
                step_ev[s][1].record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in step_ev[W:]]
    dec_ms = [dec_ev[s][0].elapsed_time(dec_ev[s][1]) for s in range(W, W + K)]
    dec_bytes = [wl.decode_bytes(s) for s in range(W, W + K)]
    total_ms = float(np.sum(step_ms))

    # --- end to end through the C ABI with host buffers: per step the H2D copies of
    # the step's inputs from pinned memory and the D2H copies of its outputs ------
    # a layer's inputs (q, k, v, modality ids) are packed in one pinned block
    # (16-byte aligned device views). The copies run on side streams: layer 0's block
    # first, the other layers' while layer 0 decodes; the outputs of all layers but
    # the last while the last decodes, then the last one's. The step's timed region
    # opens before its first input copy and closes after its last output copy.
    srcs = (wl.q, wl.k, wl.v, wl.mod)
    nl = spec.layers
    sizes = [t[0].numel() * t[0].element_size() for t in srcs]          # one step, all layers
    lsizes = [sz // nl for sz in sizes]                                   # one layer
    loffs = [0]
    for sz in lsizes[:-1]:
        loffs.append(loffs[-1] + (sz + 15) // 16 * 16)
    lbytes = (loffs[-1] + lsizes[-1] + 15) // 16 * 16
    hin = torch.empty((K, nl, lbytes), dtype=torch.uint8).pin_memory()
    for i in range(K):
        for t, o, sz in zip(srcs, loffs, lsizes):
            hin[i, :, o:o + sz].copy_(t[W + K + i].reshape(nl, -1).view(torch.uint8).cpu())
    din = torch.empty((nl, lbytes), dtype=torch.uint8, device=dev)
    dq, dk, dv, dm = ([din[l, o:o + sz].view(t.dtype).view(t.shape[2:]) for l in range(nl)]
                      for t, o, sz in zip(srcs, loffs, lsizes))
    hout = torch.empty((K,) + tuple(wl.out.shape), dtype=torch.float32).pin_memory()
    e2e_ev = [(ev(), ev()) for _ in range(K)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    sync = lambda: torch.cuda.Event()
    fork_ev, join_ev = [sync() for _ in range(K)], [sync() for _ in range(K)]
    in_ev = [[sync() for _ in range(2)] for _ in range(K)]
    out_ev = [[sync() for _ in range(2)] for _ in range(K)]

    def e2e_steps(cs):
        for i in range(K):
            flush.zero_()
            e2e_ev[i][0].record(cs)
            fork_ev[i].record(cs)
            s_in.wait_event(fork_ev[i])
            s_out.wait_event(fork_ev[i])
            with torch.cuda.stream(s_in):
                din[0].copy_(hin[i, 0], non_blocking=True)
                in_ev[i][0].record(s_in)
                if nl > 1:
                    din[1:].copy_(hin[i, 1:], non_blocking=True)
                    in_ev[i][1].record(s_in)

            def before(l, i=i):
                if l < 2:
                    cs.wait_event(in_ev[i][l])

            def after(l, i=i):
                if l < nl - 2:
                    return
                j = l - (nl - 2)  # 0: layers 0 .. nl - 2 are done; 1: the last layer
                out_ev[i][j].record(cs)
                s_out.wait_event(out_ev[i][j])
                with torch.cuda.stream(s_out):
                    if l == nl - 1:
                        hout[i, l].copy_(wl.out[l], non_blocking=True)
                    else:
                        hout[i, :l + 1].copy_(wl.out[:l + 1], non_blocking=True)

            wl.step_calls(W + K + i, dq, dk, dv, dm, cs, before=before, after=after)
            join_ev[i].record(s_out)
            cs.wait_event(join_ev[i])
            e2e_ev[i][1].record(cs)
    g2 = None
    if use_graphs:
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2, stream=stream):
            e2e_steps(torch.cuda.current_stream())
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    with torch.cuda.stream(stream):
        if use_graphs:
            g2.replay()
        else:
            e2e_steps(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = float(np.sum([a.elapsed_time(b) for a, b in e2e_ev]))
    assert torch.isfinite(hout).all(), "non-finite decode output"
    h2d = int(sum(sizes))
    d2h = int(wl.out.numel() * 4)

    # --- dense bf16 decode over the same context (comparison baseline) --------
    dense = dense_baseline(spec, wl, dev, K, W, flush, stream)

    # --- max over ranks --------------------------------------------------------
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dev, world)
    tokens = world * spec.batch * K
    value = tokens / (total_ms / 1e3)
    e2e_value = tokens / (e2e_ms / 1e3)
    avg_dec_s = float(np.mean(dec_ms)) / 1e3
    achieved = float(np.mean(dec_bytes)) / avg_dec_s / 1e9
    peak, peak_kind = peaks()
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": round(total_ms / K, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u2 codes, f32 accumulate",
            "data": "synthetic",
            "config": workload_config(spec, world, args.meta),
            "launch": {"num_splits": wl.S, "fused_append": bool(wl.fused),
                       "graph": "one CUDA graph for all steps (flush + events + C-ABI calls)" if use_graphs
                       else "eager"},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": captured_traffic(spec.name, args.meta),
                         "peak_source": peak_kind,
                         "kernel": "decode_step_kernel (append + decode launch)" if wl.fused
                         else "kv_append_kernel + decode_split_k launches",
                         "avg_launch_us": round(avg_dec_s * 1e6, 3),
                         "bytes_per_launch": int(np.mean(dec_bytes))},
            "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": wl.launches_per_step(True) * K,
            "clocks": clk,
            "dense_bf16": dense,
        }
        if not args.no_cpu_baseline and world == 1:  # the oracle is timed at N = 1 only
            line["cpu_baseline"] = cpu_baseline(spec, seed, args.meta)
        print(json.dumps(line), flush=True)
    del graph, g2
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def dense_baseline(spec, wl, dev, K, W, flush, stream):
    """The library's dense bf16 split-K decode over an unquantised cache of the
    same shape and context (random bf16 K/V), every layer, K timed steps with the
    same L2 flush; compared with the packed path's decode + combine."""
    import bit_kv_cache_pack_b200 as m
    B, H, Hq = spec.batch, spec.num_kv_heads, spec.num_q_heads
    T = wl.lengths.astype(np.int64) + W + K
    cap = int(-(-int(T.max()) // 32) * 32)
    g = torch.Generator(device=dev).manual_seed(99)
    ks, vs, qs = [], [], []
    for _ in range(spec.layers):
        ks.append(torch.randn(B, H, cap, 128, generator=g, device=dev).to(torch.bfloat16))
        vs.append(torch.randn(B, H, cap, 128, generator=g, device=dev).to(torch.bfloat16))
        qs.append(torch.randn(B, Hq, 128, generator=g, device=dev).to(torch.bfloat16))
    lens = torch.as_tensor(T, dtype=torch.int32, device=dev)
    S = 0
    part = torch.empty(m.omnikv_dense_partials_bytes(B, Hq, 4096) // 4, device=dev)
    out = torch.empty(spec.layers, B, Hq, 128, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def step(st):
        for layer in range(spec.layers):
            m.omnikv_dense_decode_bf16(ks[layer], vs[layer], lens, B, Hq, H, cap, int(T.max()), qs[layer], part, S,
                                       out[layer], err, st)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step(torch.cuda.current_stream())
    times = []
    with torch.cuda.stream(stream):
        for i in range(W + K):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
            times.append((e0, e1))
    torch.cuda.synchronize(dev)
    ms = float(np.mean([a.elapsed_time(b) for a, b in times[W:]]))
    assert int(err.item()) == 0 and torch.isfinite(out).all()
    bytes_step = spec.layers * (int(T.sum()) * H * 512 + B * Hq * 128 * 2)
    del graph
    return {"ms_per_step": round(ms, 4), "us_per_layer": round(ms * 1e3 / spec.layers, 3),
            "tokens_per_s": round(B / (ms / 1e3), 3), "achieved_GBps": round(bytes_step / (ms / 1e3) / 1e9, 1),
            "bytes_per_token_head": 512, "what": "decode attention only (no cache append), same context, bf16 K/V"}


# ----------------------------------------------------------------------------
# the CPU oracle, timed (baseline and reference arm)
# ----------------------------------------------------------------------------
def host_info():
    """Host cores and CPU model of the machine the oracle is timed on."""
    model = ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


class OneCore:
    """Context: the oracle runs on one host core -- BLAS / OpenMP pools limited to
    one thread, torch's intra-op pool to one thread, and the process pinned to a
    single CPU of its allowed set -- restored on exit."""

    def __enter__(self):
        import threadpoolctl
        self.limits = threadpoolctl.threadpool_limits(1)
        self.threads = torch.get_num_threads()
        torch.set_num_threads(1)
        self.aff = os.sched_getaffinity(0)
        os.sched_setaffinity(0, {min(self.aff)})
        return self

    def __exit__(self, *exc):
        os.sched_setaffinity(0, self.aff)
        torch.set_num_threads(self.threads)
        self.limits.restore_original_limits()
        return False


def oracle_sample_shape(spec):
    """Layers and sequences of the workload the oracle is timed on: all of it when
    one layer holds at most ~100k token-heads, else one layer and up to 4 sequences
    (the oracle decodes ~1 s per 65,536-token sequence and kv-head set)."""
    from synth.workloads import seq_lengths
    per_layer = int(seq_lengths(spec, 0).astype(np.int64).sum()) * spec.num_kv_heads
    if per_layer <= 100_000:
        return min(spec.layers, 12), spec.batch
    return 1, min(spec.batch, 4)


def _oracle_sequences(spec, seed, layers, seqs, extra_steps, meta="fp16"):
    """The oracle's caches of the sampled (layer, sequence) pairs, each a batch-1
    cache prefilled with that sequence's context (untimed), and every layer's
    decode inputs for extra_steps steps."""
    from oracle import codec
    from synth.workloads import codebook, decode_inputs, key_drift, layer_params, prefill_inputs, seq_lengths
    L = seq_lengths(spec, seed)
    cap = int(-(-(int(L.max()) + extra_steps) // 32) * 32)
    out = []
    for layer in layers:
        params = layer_params(spec, seed, layer)
        ocfg = codec.OracleConfig(codebook(spec.key_bits), codebook(spec.value_bits),
                                  params["key_signs"].numpy(), params["value_rot"].numpy(),
                                  spec.num_q_heads, spec.num_kv_heads)
        drift = key_drift(spec, seed, layer, cap // 32, "cpu")
        caches = []
        for b in seqs:
            k, v, mod = prefill_inputs(spec, seed, layer, params, drift, L, "cpu", batch_index=[b])
            n = int(L[b])
            oc = codec.OracleCache(1, spec.num_kv_heads, cap, spec.key_bits, spec.value_bits, meta_format=meta)
            codec.write_cache(ocfg, oc, k[:, :, :n].numpy(), v[:, :, :n].numpy(), mod[:, :n].numpy())
            caches.append(oc)
            del k, v, mod
        steps = [decode_inputs(spec, seed, layer, s, params, drift, L + s, "cpu") for s in range(extra_steps)]
        out.append((ocfg, caches, steps))
    return out


def _oracle_step(ocfg, oc, inputs, b, num_splits=4):
    """One decode step of sequence b through the oracle: append its token, then
    the fused split-K decode and combine."""
    from oracle import codec
    from oracle.attention import decode_fused
    q, kn, vn, mn = (x[b:b + 1].numpy() for x in inputs)
    codec.write_cache(ocfg, oc, kn, vn, mn)
    return decode_fused(ocfg, oc, q, num_splits)


def cpu_baseline(spec, seed, meta="fp16"):
    """The oracle as it stands (numpy fp64, one pinned core) on a bounded sample of
    the workload -- one decode step of the sampled layers and sequences -- scaled
    linearly to the whole step (all layers, all sequences)."""
    n_layers, n_seq = oracle_sample_shape(spec)
    prepared = _oracle_sequences(spec, seed, range(n_layers), range(n_seq), 1, meta)
    with OneCore():
        t0 = time.perf_counter()
        for ocfg, caches, steps in prepared:
            for b, oc in enumerate(caches):
                _oracle_step(ocfg, oc, steps[0], b)
        dt = time.perf_counter() - t0
    scale = (spec.layers / n_layers) * (spec.batch / n_seq)
    per_step = dt * scale
    d = {"value": round(spec.batch / per_step, 6), "unit": UNIT, "cores": 1, "kind": "oracle",
         "sample": "1 decode step (append + fused decode + combine, numpy fp64) of %d of %d layers x %d of %d "
                   "sequences, %.1f s of CPU on one pinned core, scaled x%g to the whole step"
                   % (n_layers, spec.layers, n_seq, spec.batch, dt, scale),
         "extrapolated": scale != 1.0}
    d.update(host_info())
    return d


def run_reference(args):
    """The reference arm: the oracle, timed on the host. Each timed step is one
    (layer, sequence) sample of the workload's decode step (append + fused decode +
    combine), rotating over the sampled sequences; the full step's time is that
    sample's mean time x layers x sequences."""
    from synth.workloads import WORKLOADS
    world, rank, _ = dist_env()
    if rank != 0:
        return
    spec = WORKLOADS[args.workload]
    seed = WORKLOADS_KEYS.index(args.workload)
    K, W = args.steps, args.warmup
    n_seq = min(spec.batch, 2)
    prepared = _oracle_sequences(spec, seed, [0], range(n_seq), (W + K) // n_seq + 2, args.meta)
    ocfg, caches, steps = prepared[0]
    times = []
    with OneCore():
        for s in range(W + K):
            b = s % n_seq
            t0 = time.perf_counter()
            _oracle_step(ocfg, caches[b], steps[s // n_seq], b)
            if s >= W:
                times.append(time.perf_counter() - t0)
    sample_s = float(np.mean(times))
    scale = spec.layers * spec.batch
    per_step = sample_s * scale
    value = spec.batch / per_step
    base = {"value": round(value, 6), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": "each timed step: one layer's decode step (append + fused decode + combine, numpy fp64) "
                      "of one of %d sequences, on one pinned core; the whole step = x%d (%d layers x %d "
                      "sequences)" % (n_seq, scale, spec.layers, spec.batch),
            "extrapolated": scale != 1}
    base.update(host_info())
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": round(per_step * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic",
        "config": workload_config(spec, world, args.meta),
        "extrapolated": scale != 1, "sample_ms_per_step": round(sample_s * 1e3, 3),
        "cpu_baseline": base,
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_layer(args):
    """One layer of --workload: the prefill cache write of the whole batch, or
    decode + combine over that cache (split counts from --splits), each timed
    with CUDA events after warm-up, L2 flushed before every timed call. Bytes:
    write 512 B of fp16 K and V in + the packed record out per token and kv head;
    decode the packed records per token and kv head + 1 modality byte per token."""
    import dataclasses
    import bit_kv_cache_pack_b200 as m
    from synth.workloads import (WORKLOADS, codebook, key_drift, layer_params, prefill_inputs, seq_lengths,
                                 with_bits)
    spec = WORKLOADS[args.workload]
    bits = args.bits or spec.key_bits
    spec = with_bits(spec, bits, bits)
    if args.batch:
        spec = dataclasses.replace(spec, batch=args.batch)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    seed = 7
    L = seq_lengths(spec, seed)
    T = int(L.max())
    cap = int(-(-(T + 8) // 32) * 32)
    params = layer_params(spec, seed, 0)
    fmt = META_FORMATS[args.meta]
    consts = m.LayerConstants(codebook(bits), codebook(bits), params["key_signs"], params["value_rot"],
                              spec.num_q_heads, dev, key_meta_format=fmt)
    drift = key_drift(spec, seed, 0, cap // 32, dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    per_token = BYTES_PER_TOKEN_HEAD[(bits, bits, args.meta)]
    peak, _ = peaks()
    iters, warm = 5, 2

    def timed(fn, prep=None):
        ts = []
        for it in range(iters + warm):
            if prep is not None:
                prep()
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize(dev)
            if it >= warm:
                ts.append(e0.elapsed_time(e1) * 1e3)
        return float(np.median(ts))

    if args.layer == "calibrate":
        # one (layer, kv head): the first sequence's values, weights from 4 decode queries
        k, v, mod = prefill_inputs(dataclasses.replace(spec, batch=1), seed, 0, params, drift, np.array([T]), dev)
        vals = v[0, 0].contiguous()
        wts = torch.rand(T, generator=torch.Generator(device=dev).manual_seed(seed), device=dev)
        ws = torch.empty(m.omnikv_calibrate_workspace_bytes(T) // 8 + 1, dtype=torch.float64, device=dev)
        bases = torch.empty(3, 128, 128, dtype=torch.float32, device=dev)
        lam = torch.empty(3, 128, dtype=torch.float64, device=dev)
        mod0 = mod[0].contiguous()
        us = timed(lambda: m.omnikv_calibrate_bases(vals, mod0, wts, T, ws, bases, lam))
        gram_flop = 2.0 * T * 128 * 128  # each token's weighted outer product, fp64
        fp64_peak = 148 * 64 * 2 * 1.965e9 / 1e12  # SMs x fp64 FMA lanes x 2 flop x max SM clock (TFLOP/s)
        print(json.dumps({"layer": "calibrate", "workload": spec.name, "tokens": T, "us": round(us, 2),
                          "gram_gflop": round(gram_flop / 1e9, 3),
                          "fp64_tflops_over_whole_call": round(gram_flop / (us * 1e-6) / 1e12, 3),
                          "fp64_peak_tflops_derived": round(fp64_peak, 1)}), flush=True)
        return
    if args.layer == "write":
        k, v, mod = prefill_inputs(spec, seed, 0, params, drift, np.full(spec.batch, T), dev)
        c = m.KVCache(spec.batch, spec.num_kv_heads, cap, bits, bits, dev, key_meta_format=fmt)

        def empty():  # the prefill of an empty cache, every time
            c.seq_lens.zero_()
            c.struct.max_seq_len = 0

        us = timed(lambda: m.omnikv_write_cache(consts.struct, c.struct, k, v, mod, T), empty)
        byts = int(spec.batch * T * spec.num_kv_heads * (512 + per_token) + spec.batch * T)
        print(json.dumps({"layer": "write", "workload": spec.name, "meta": args.meta, "tokens": spec.batch * T, "us": round(us, 2),
                          "GBps": round(byts / us / 1e3, 1), "frac": round(byts / us / 1e3 / peak, 4),
                          "error_word": int(c.error_word.item())}), flush=True)
        return
    cache = m.KVCache(spec.batch, spec.num_kv_heads, cap, bits, bits, dev, key_meta_format=fmt)
    rings = m.stream_rings(spec.batch, spec.num_kv_heads, dev) if args.stream else None
    for b in range(spec.batch):
        k, v, mod = prefill_inputs(spec, seed, 0, params, drift, L, dev, batch_index=[b])
        n = int(L[b])
        if rings is not None:
            m.omnikv_stream_write_cache(consts.struct, cache.sequence_view(b), rings[0][b:b + 1], rings[1][b:b + 1],
                                        k[:, :, :n].contiguous(), v[:, :, :n].contiguous(), mod[:, :n].contiguous(), n)
        else:
            m.omnikv_write_cache(consts.struct, cache.sequence_view(b), k[:, :, :n].contiguous(),
                                 v[:, :, :n].contiguous(), mod[:, :n].contiguous(), n)
        del k, v, mod
    cache.struct.max_seq_len = T
    q = torch.randn(spec.batch, spec.num_q_heads, 128, device=dev).half()
    byts = int(int(L.astype(np.int64).sum()) * spec.num_kv_heads * per_token + int(L.sum()))
    for S in [int(x) for x in args.splits.split(",")]:
        S = S or m.omnikv_default_splits(consts.struct, cache.struct)
        part = m.partials_tensor(spec.batch, spec.num_q_heads, S, dev)
        out = torch.empty(spec.batch, spec.num_q_heads, 128, device=dev)
        dec = timed(lambda: m.omnikv_decode_attention(consts.struct, cache.struct, q, part, S))
        comb = timed(lambda: m.omnikv_combine(consts.struct, cache.struct, part, S, out))
        print(json.dumps({"layer": "decode", "workload": spec.name, "meta": args.meta, "splits": S, "decode_us": round(dec, 2),
                          "combine_us": round(comb, 2), "GBps": round(byts / dec / 1e3, 1),
                          "frac": round(byts / dec / 1e3 / peak, 4), "error_word": int(cache.error_word.item())}),
              flush=True)
        if rings is not None:
            part2 = m.partials_tensor(spec.batch, spec.num_q_heads, S + m._abi.OMNIKV_STREAM_TAIL_SPLITS, dev)
            st = timed(lambda: m.omnikv_stream_decode(consts.struct, cache.struct, rings[0], rings[1], q, part2, S, out))
            print(json.dumps({"layer": "stream-decode", "workload": spec.name, "meta": args.meta, "splits": S,
                              "us": round(st, 2), "vs_decode_plus_combine": round(st / (dec + comb), 3),
                              "what": "packed body + tail kernel (newest <= 159 positions, 4 CTAs per kv head) + combine, 3 launches"}),
                  flush=True)


def main():
    args = parse_args()
    if args.layer:
        run_layer(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
