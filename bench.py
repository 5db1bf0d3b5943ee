"""Benchmark of the BlockFFN chunk-layer forward on B200.

One step = one pass of the hot path over one batch of synthetic input: `chunks` chunk forwards
(router + chunk union + sparse experts) through the C ABI, chunk c using weight replica c % replicas.
Decode chunks of up to 8 tokens go through one batched call per step (two launches: the router of
every chunk, then a persistent expert kernel whose SMs form K = --streams teams, team k taking chunks
k, k + K, ...).  With --mode streams (and for longer chunks) chunk c is issued on stream c % K with
its own workspace and the concurrency hint, so K chunks run side by side, each on 1/K of the SMs.
Decode lines also time one chunk at a time on the whole GPU (roofline.single_chunk).  The replicas
stand for distinct layers of a stacked model and keep
the weights (16 x 128 MiB for the default workload) well above the 126 MB L2, so every chunk streams
its active experts from HBM ("inputs larger than L2").  A step is captured once into a CUDA graph
and replayed; time is taken with CUDA events on the replay stream, with a barrier and a
synchronize on both sides, max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode] [--impl ours|reference]

--impl reference times the fp64 CPU oracle (the reference implementation of this build) on the
host cores on a bounded sample of the same workload.  Multi-GPU runs (torchrun) shard chunks across
ranks with no collective in the data path (weak scaling).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "BlockFFN layer tokens/s at chunk L=8 and achieved HBM GB/s over active bytes"
METRIC_PREFILL = "BlockFFN layer tokens/s on a prefill chunk and achieved TFLOP/s (tcgen05 grouped GEMMs)"
DECODE_MAX_L = 32
FALLBACK_HBM_GBS = 6650.0


# ---------------------------------------------------------------------------------- helpers
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def shard_seed(seed: int, rank: int) -> int:
    """Chunk stream of a rank: every rank draws its own chunks (weak scaling)."""
    return seed * 1000003 + rank


def reduce_max(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def measured_peaks(key="hbm_gbs"):
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j[key]), "measured"
    except Exception:
        return (FALLBACK_HBM_GBS if key == "hbm_gbs" else 1590.0), "fallback"


# the sources the batched decode kernels are compiled from (the kernels, the headers they include, the
# host code that sizes their launches); a change to any of them makes recorded counters stale
BATCH_KERNEL_SOURCES = ("api.cu", "decode_batch.cu", "blockffn_internal.cuh", "ptx.cuh")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "chunk_sparse_moe_router_b200", "csrc")
    for name in BATCH_KERNEL_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic_ratio(workload_name: str):
    """DRAM bytes per algorithmic (active) byte from the committed ncu summary, only if the kernel
    sources are unchanged since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            j = json.load(f)
        rec = j.get(workload_name)
        if rec and rec.get("kernel_source_hash") == kernel_source_hash():
            return float(rec["dram_bytes_per_active_byte"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"bffn_clocks_{os.getpid()}_{gpu_index}.csv")

    def __enter__(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.25)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 8:
                    rows.append(parts)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        pw = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "power_w_max": max(pw) if pw else None}


# ---------------------------------------------------------------------------------- workload
def prefill_flops(d, E, de, L, pairs):
    """Algorithmic FLOPs of a prefill chunk: both expert projections over the (token, expert) pairs
    with r > 0, plus the router projection."""
    return 4.0 * d * de * pairs + 2.0 * L * d * E


def active_bytes(d, E, de, L, n_active):
    """Algorithmic bytes of one chunk: router weights, gain and bias, x in, y out, and W1_i + W2_i of
    every expert in the chunk's union (bf16)."""
    return 4 * d * E + 4 * E * 2 + 2 * L * d + 4 * L * d + n_active * (2 * d * de * 2)


def build_inputs(w, rank, device, chunks):
    """The workload's weight replicas stacked one after another on the device (W1 [R, E, de, d] and so
    on, the layout the batched call takes; layers[r] holds views of replica r for the per-chunk call),
    and the chunks on the host: chunk c uses replica c % R."""
    import numpy as np
    import torch

    import gen

    R, d, E, de = w.replicas, w.d, w.E, w.de
    stack = {"Wr": torch.empty((R, d, E), dtype=torch.float32, device=device),
             "br": torch.empty((R, E), dtype=torch.float32, device=device),
             "g": torch.empty((R, E), dtype=torch.float32, device=device),
             "W1": torch.empty((R, E, de, d), dtype=torch.bfloat16, device=device),
             "W2": torch.empty((R, E, d, de), dtype=torch.bfloat16, device=device)}
    layers = []
    host_x = []
    per = (chunks + R - 1) // R
    for r in range(R):
        lay = w.layer(r)
        stack["Wr"][r].copy_(torch.from_numpy(lay.Wr))
        stack["br"][r].copy_(torch.from_numpy(lay.br))
        stack["g"][r].copy_(torch.from_numpy(lay.g))
        stack["W1"][r].view(torch.int16).copy_(torch.from_numpy(lay.W1.view(np.int16)))
        stack["W2"][r].view(torch.int16).copy_(torch.from_numpy(lay.W2.view(np.int16)))
        layers.append({"lay": lay if r == 0 else None, **{k: v[r] for k, v in stack.items()}})
        host_x.append(gen.make_chunks(shard_seed(w.seed, rank), lay, per, w.L, w.noise, stream=r))
        del lay
    # chunk c -> replica c % R, position c // R within that replica's stream
    x_all = np.empty((chunks, w.L, w.d), dtype=np.uint16)
    for c in range(chunks):
        x_all[c] = host_x[c % R][c // R]
    return layers, stack, x_all


# ---------------------------------------------------------------------------------- our arm
def run_ours(args, w):
    import numpy as np
    import torch
    import torch.distributed as dist

    import chunk_sparse_moe_router_b200 as bffn

    world, rank, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        dist.init_process_group("nccl", device_id=device,
                                timeout=__import__("datetime").timedelta(seconds=120))

    chunks = args.chunks or w.n_chunks
    t_gen = time.time()
    layers, stack, x_host_np = build_inputs(w, rank, device, chunks)
    gen_s = time.time() - t_gen
    L, d, E, de = w.L, w.d, w.E, w.de
    x_dev = torch.from_numpy(x_host_np.view(np.int16)).to(device).view(torch.bfloat16)
    y = torch.empty((chunks, L, d), dtype=torch.float32, device=device)
    idx = torch.empty((chunks, E), dtype=torch.int32, device=device)
    nact = torch.empty((chunks,), dtype=torch.int32, device=device)
    cnts = torch.empty((chunks, 2), dtype=torch.int32, device=device)  # TLS / CLS zero counts

    # Decode chunks of up to 8 tokens (default): the batched call, all chunks of a step in two launches,
    # the SMs in K teams (--streams), team k taking chunks k, k + K, ...; chunk c uses replica c % R.
    # Otherwise (--mode streams, longer chunks, prefill): K streams, each with its own workspace: chunk c
    # goes to stream c % K, and with K > 1 each call takes 1/K of the SMs, so K chunks run side by side.
    batched = args.mode == "batch" and L <= 8
    K = max(1, args.streams if L <= DECODE_MAX_L else 1)
    flags = bffn.BFFN_FLAGS_SHARE(K) if K > 1 else 0
    if batched:
        ws_bytes = bffn.blockffn_batch_workspace_size(chunks, L, d, E, de, flags)
        workspaces = [torch.zeros(ws_bytes, dtype=torch.uint8, device=device)]
    else:
        ws_bytes = bffn.blockffn_workspace_size(L, d, E, de)
        workspaces = [bffn.new_workspace(L, d, E, de, device) for _ in range(K)]  # zero-filled
    ws_ptrs = [t.data_ptr() for t in workspaces]
    bufs = [(x_dev, y, idx, nact, cnts)]  # a second set is added for the end-to-end pipeline

    def step(streams, buf=None):
        x_dev, y, idx, nact, cnts = buf if buf is not None else bufs[0]
        if batched:
            rc = bffn.blockffn_chunk_forward_batch(
                x_dev.data_ptr(), chunks, L, d, None, w.replicas, stack["Wr"].data_ptr(), stack["g"].data_ptr(),
                stack["br"].data_ptr(), stack["W1"].data_ptr(), stack["W2"].data_ptr(), E, de, y.data_ptr(),
                idx.data_ptr(), nact.data_ptr(), cnts.data_ptr(), None, flags, ws_ptrs[0], ws_bytes,
                streams[0].cuda_stream)
            if rc != 0:
                raise bffn.BlockFFNError(rc, "blockffn_chunk_forward_batch")
            return
        if K > 1:  # fork: the side streams start after everything queued on the main one
            ev = torch.cuda.Event()
            ev.record(streams[0])
            for sk in streams[1:]:
                sk.wait_event(ev)
        for c in range(chunks):
            lay = layers[c % w.replicas]
            k = c % K
            rc = bffn.blockffn_chunk_forward_ex(
                x_dev[c].data_ptr(), L, d, lay["Wr"].data_ptr(), lay["g"].data_ptr(), lay["W1"].data_ptr(),
                lay["W2"].data_ptr(), E, de, y[c].data_ptr(), idx[c].data_ptr(), nact[c:].data_ptr(),
                lay["br"].data_ptr(), None, cnts[c].data_ptr(), None, flags, ws_ptrs[k], ws_bytes,
                streams[k].cuda_stream)
            if rc != 0:
                raise bffn.BlockFFNError(rc, "blockffn_chunk_forward_ex")
        if K > 1:  # join
            for sk in streams[1:]:
                ev = torch.cuda.Event()
                ev.record(sk)
                streams[0].wait_event(ev)

    s = torch.cuda.Stream(device)
    side = [torch.cuda.Stream(device) for _ in range(0 if batched else K - 1)]
    streams = [s] + side
    with torch.cuda.stream(s):
        step(streams)
        s.synchronize()
        for ws in workspaces:
            if bffn.device_status(workspace=ws, stream=s.cuda_stream) != 0:
                raise RuntimeError("device-side wait ran out")
        graph = torch.cuda.CUDAGraph()
        graph.capture_begin()
        step(streams)
        graph.capture_end()
        s.synchronize()
        for _ in range(args.warmup):
            graph.replay()
        s.synchronize()

        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(device)
        torch.cuda.synchronize(device)
        with ClockSampler(local) as clk:
            e0.record(s)
            for _ in range(args.steps):
                graph.replay()
            e1.record(s)
            e1.synchronize()
        torch.cuda.synchronize(device)
        barrier(device)
        t_ms = e0.elapsed_time(e1)
        for ws in workspaces:
            if bffn.device_status(workspace=ws, stream=s.cuda_stream) != 0:
                raise RuntimeError("device-side wait ran out during the timed region")

        # end to end, as a serving loop runs it: every step copies its x in from pinned host memory and its
        # y and active sets back out, double-buffered on two copy streams, so that step k+1's input and step
        # k-1's results cross PCIe while step k computes
        x_pin = torch.from_numpy(x_host_np.view(np.int16)).pin_memory()
        bufs.append((torch.empty_like(x_dev), torch.empty_like(y), torch.empty_like(idx), torch.empty_like(nact),
                     torch.empty_like(cnts)))
        graphs = [graph, torch.cuda.CUDAGraph()]
        step(streams, bufs[1])
        s.synchronize()
        graphs[1].capture_begin()
        step(streams, bufs[1])
        graphs[1].capture_end()
        pins = [(torch.empty(y.shape, dtype=y.dtype).pin_memory(), torch.empty(idx.shape, dtype=idx.dtype).pin_memory(),
                 torch.empty(nact.shape, dtype=nact.dtype).pin_memory()) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(k):
            b = k % 2
            xb, yb, ib, nb, _ = bufs[b]
            if k >= 2:  # buffer b's previous input has been consumed
                s_in.wait_event(ev_done[b])
            with torch.cuda.stream(s_in):
                xb.view(torch.int16).copy_(x_pin, non_blocking=True)
            ev_in[b].record(s_in)
            s.wait_event(ev_in[b])
            if k >= 2:  # buffer b's previous results have left the device
                s.wait_event(ev_out[b])
            graphs[b].replay()
            ev_done[b].record(s)
            s_out.wait_event(ev_done[b])
            with torch.cuda.stream(s_out):
                pins[b][0].copy_(yb, non_blocking=True)
                pins[b][1].copy_(ib, non_blocking=True)
                pins[b][2].copy_(nb, non_blocking=True)
            ev_out[b].record(s_out)

        def run(n):  # n pipelined steps between events on s (the copy streams start after the first)
            start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            start.record(s)
            s_in.wait_event(start)
            s_out.wait_event(start)
            for k in range(n):
                e2e_step(k)
            for b in range(2):
                s.wait_event(ev_out[b])
            end.record(s)
            end.synchronize()
            return start, end

        run(2)
        torch.cuda.synchronize(device)
        barrier(device)
        torch.cuda.synchronize(device)
        e2e_steps = max(3, args.steps // 2)
        f0, f1 = run(e2e_steps)
        barrier(device)
        e2e_ms = f0.elapsed_time(f1)
        last = pins[(e2e_steps - 1) % 2]
        if not (torch.equal(last[0], y.cpu()) and torch.equal(last[2], nact.cpu())):
            raise RuntimeError("the pipelined end-to-end results differ from the device-timed step's")
        del graphs

        # one chunk at a time on the whole GPU (the latency a verification step sees per layer): the
        # first n1 chunks through the per-chunk entry point on one stream, as one graph
        single = None
        if L <= DECODE_MAX_L:
            n1 = min(chunks, 512)
            ws1 = bffn.new_workspace(L, d, E, de, device)
            ws1_bytes = bffn.blockffn_workspace_size(L, d, E, de)
            y1 = torch.empty((n1, L, d), dtype=torch.float32, device=device)
            i1 = torch.empty((n1, E), dtype=torch.int32, device=device)
            c1 = torch.empty((n1, 2), dtype=torch.int32, device=device)
            n1a = torch.empty((n1,), dtype=torch.int32, device=device)

            def single_step():
                for c in range(n1):
                    lay = layers[c % w.replicas]
                    rc = bffn.blockffn_chunk_forward_ex(
                        x_dev[c].data_ptr(), L, d, lay["Wr"].data_ptr(), lay["g"].data_ptr(), lay["W1"].data_ptr(),
                        lay["W2"].data_ptr(), E, de, y1[c].data_ptr(), i1[c].data_ptr(), n1a[c:].data_ptr(),
                        lay["br"].data_ptr(), None, c1[c].data_ptr(), None, 0, ws1.data_ptr(), ws1_bytes,
                        s.cuda_stream)
                    if rc != 0:
                        raise bffn.BlockFFNError(rc, "blockffn_chunk_forward_ex")

            single_step()
            s.synchronize()
            g1 = torch.cuda.CUDAGraph()
            g1.capture_begin()
            single_step()
            g1.capture_end()
            for _ in range(3):
                g1.replay()
            s.synchronize()
            h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 5
            h0.record(s)
            for _ in range(reps):
                g1.replay()
            h1.record(s)
            h1.synchronize()
            if bffn.device_status(workspace=ws1, stream=s.cuda_stream) != 0:
                raise RuntimeError("device-side wait ran out (single-chunk timing)")
            us1 = h0.elapsed_time(h1) * 1e3 / (reps * n1)
            b1 = float(sum(active_bytes(d, E, de, L, int(n)) for n in n1a.cpu().numpy())) / n1
            single = {"us_per_chunk": round(us1, 3), "tokens_per_s": round(L / (us1 * 1e-6), 1),
                      "achieved_gbs": round(b1 / (us1 * 1e-6) / 1e9, 1), "chunks": n1,
                      "entry_point": "blockffn_chunk_forward_ex, whole GPU, one chunk at a time"}
            del g1

    t_max = reduce_max(t_ms, device)
    e2e_max = reduce_max(e2e_ms, device)
    n_act_host = nact.cpu().numpy()
    pairs_host = L * E - cnts[:, 0].cpu().numpy().astype(np.int64)
    prefill = L > DECODE_MAX_L
    total_active = float(sum(active_bytes(d, E, de, L, int(n)) for n in n_act_host))
    ms_per_step = t_max / args.steps
    tokens_step = chunks * L * world
    value = tokens_step / (ms_per_step * 1e-3)
    achieved_gbs = total_active / (ms_per_step * 1e-3) / 1e9  # per GPU: every rank streams its own
    peak, peak_kind = measured_peaks()
    ratio = recorded_traffic_ratio(w.name + ("/batch" if batched else "/streams"))
    traffic = None if ratio is None else ratio * total_active / chunks
    if prefill:
        flops = float(sum(prefill_flops(d, E, de, L, int(p)) for p in pairs_host))
        achieved_tf = flops / (ms_per_step * 1e-3) / 1e12
        tpeak, tpeak_kind = measured_peaks("bf16_tflops")
        roofline = {"bound": "tensor", "achieved": round(achieved_tf, 1), "peak": tpeak, "unit": "TFLOP/s",
                    "frac": round(achieved_tf / tpeak, 4), "peak_kind": tpeak_kind + " (bf16 burst)",
                    "kernel": "one prefill chunk forward (router, grouping, tcgen05 GEMM1 and GEMM2)",
                    "flops_per_chunk": round(flops / chunks, 1),
                    "pairs_per_chunk": round(float(pairs_host.mean()), 1),
                    "us_per_chunk": round(ms_per_step * 1e3 / chunks, 3), "traffic": None}
    else:
        kname = ("batch_expert_kernel + batch_router_kernel: every chunk of the step in two launches (time "
                 "of both counted)" if batched else "expert_decode_kernel: one chunk forward, router included")
        roofline = {"bound": "hbm", "achieved": round(achieved_gbs, 1), "peak": peak, "unit": "GB/s",
                    "frac": round(achieved_gbs / peak, 4), "peak_kind": peak_kind, "kernel": kname,
                    "bytes_per_chunk": round(total_active / chunks, 1),
                    "us_per_chunk": round(ms_per_step * 1e3 / chunks, 3),
                    "traffic": None if traffic is None else round(traffic, 1)}
        if single is not None:
            single["frac"] = round(single["achieved_gbs"] / peak, 4)
            roofline["single_chunk"] = single
    out = {
        "metric": METRIC_PREFILL if prefill else METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {**w.describe(), "chunks_per_step": chunks,
                   "l2": f"inputs larger than L2: {w.replicas} weight replicas, "
                         f"{w.replicas * E * 2 * d * de * 2 / 1e9:.2f} GB of expert weights",
                   "mean_n_active": round(float(n_act_host.mean()), 3),
                   "cls": round(1.0 - float(n_act_host.mean()) / E, 4),
                   "parallelism": f"dp{world} (chunks sharded, no collective in the data path)",
                   "mode": "batch" if batched else "streams",
                   "concurrent_chunks": K},
        "roofline": roofline,
        "e2e": {"value": round(tokens_step / (e2e_max / e2e_steps * 1e-3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": int(x_host_np.nbytes),
                "d2h_bytes_per_step": int(y.numel() * 4 + idx.numel() * 4 + nact.numel() * 4),
                "steps": e2e_steps,
                "pipeline": "double-buffered: step k+1's x in and step k-1's results out overlap step k"},
        "gpu_launches": (2 if batched else (7 if prefill else 1) * chunks) * args.steps,
        "clocks": clk.summary(),
        "gen_seconds": round(gen_s, 1),
    }
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, layers[0]["lay"], x_host_np, args.cpu_seconds,
                                           y_gpu=y, n_gpu=n_act_host)
    if rank == 0:
        print(json.dumps(out), flush=True)
    del graph
    if world > 1:
        dist.destroy_process_group()


# ---------------------------------------------------------------------------------- sparsity sweep
def run_tls_sweep(args):
    """Config 4 of the measurement plan: a stacked model FFN of `--replicas` layers (default 32: d=4096,
    E=128, de=256, 17.2 GB of bf16 expert weights), L=8 chunks, one batched call per step through all
    layers (chunk c on layer c % layers).  The router bias is set per point for token-level sparsity
    TLS in --tls-list, the chunk-level sparsity is measured, and a dense point forces every expert
    active (bias +50) on the same layers, through the same kernels.  One JSON line per point; the
    sparse points carry their speedup over the dense point next to the bound 1 / (1 - CLS)."""
    import numpy as np
    import torch

    import chunk_sparse_moe_router_b200 as bffn
    import gen

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    base = gen.workload("tls_sweep")
    R = args.replicas or base.replicas
    d, E, de, L = base.d, base.E, base.de, base.L
    C = args.chunks or 8 * R
    K = args.streams
    t_gen = time.time()
    W1 = torch.empty((R, E, de, d), dtype=torch.bfloat16, device=device)
    W2 = torch.empty((R, E, d, de), dtype=torch.bfloat16, device=device)
    Wr = torch.empty((R, d, E), dtype=torch.float32, device=device)
    g = torch.empty((R, E), dtype=torch.float32, device=device)
    host = []  # per layer: Wr (for the bias scale and the margin test)
    for r in range(R):
        lay = base.layer(r)
        W1[r].view(torch.int16).copy_(torch.from_numpy(lay.W1.view(np.int16)))
        W2[r].view(torch.int16).copy_(torch.from_numpy(lay.W2.view(np.int16)))
        Wr[r].copy_(torch.from_numpy(lay.Wr))
        g[r].copy_(torch.from_numpy(lay.g))
        lay.W1 = lay.W2 = None
        host.append(lay)
    gen_s = time.time() - t_gen
    peak, peak_kind = measured_peaks()
    points = [p.strip() for p in args.tls_list.split(",")]
    # the dense point first, so that every sparse line can quote its speedup over it
    points = ["dense"] + [p for p in points if p != "dense"]
    flags = bffn.BFFN_FLAGS_SHARE(K)
    ws_bytes = bffn.blockffn_batch_workspace_size(C, L, d, E, de, flags)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=device)
    y = torch.empty((C, L, d), dtype=torch.float32, device=device)
    idx = torch.empty((C, E), dtype=torch.int32, device=device)
    nact = torch.empty((C,), dtype=torch.int32, device=device)
    cnts = torch.empty((C, 2), dtype=torch.int32, device=device)
    dense_tps = None
    s = torch.cuda.Stream(device)
    for pt in points:
        dense = pt == "dense"
        tls = 0.5 if dense else float(pt)
        beta = gen.beta_for_tls(tls)
        br = torch.empty((R, E), dtype=torch.float32, device=device)
        per = C // R
        x_host = np.empty((C, L, d), dtype=np.uint16)
        for r in range(R):
            lay = host[r]
            sigma = np.sqrt(lay.var_x * np.sum(lay.Wr.astype(np.float64) ** 2, axis=0))
            lay.br = np.full(E, 50.0, np.float32) if dense else (-beta * sigma).astype(np.float32)
            br[r].copy_(torch.from_numpy(lay.br))
            xs = gen.make_chunks(base.seed, lay, per, L, base.noise, stream=r)
            for q in range(per):
                x_host[q * R + r] = xs[q]
        x = torch.from_numpy(x_host.view(np.int16)).to(device).view(torch.bfloat16)

        def step():
            rc = bffn.blockffn_chunk_forward_batch(
                x.data_ptr(), C, L, d, None, R, Wr.data_ptr(), g.data_ptr(), br.data_ptr(), W1.data_ptr(),
                W2.data_ptr(), E, de, y.data_ptr(), idx.data_ptr(), nact.data_ptr(), cnts.data_ptr(), None, flags,
                ws.data_ptr(), ws_bytes, s.cuda_stream)
            if rc != 0:
                raise bffn.BlockFFNError(rc, "blockffn_chunk_forward_batch")

        with torch.cuda.stream(s):
            step()
            s.synchronize()
            if bffn.device_status(workspace=ws, stream=s.cuda_stream) != 0:
                raise RuntimeError("device-side wait ran out")
            graph = torch.cuda.CUDAGraph()
            graph.capture_begin()
            step()
            graph.capture_end()
            for _ in range(args.warmup):
                graph.replay()
            s.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with ClockSampler(0) as clk:
                e0.record(s)
                for _ in range(args.steps):
                    graph.replay()
                e1.record(s)
                e1.synchronize()
            if bffn.device_status(workspace=ws, stream=s.cuda_stream) != 0:
                raise RuntimeError("device-side wait ran out during the timed region")
            del graph
        ms = e0.elapsed_time(e1) / args.steps
        n_host = nact.cpu().numpy()
        zeros = cnts[:, 0].cpu().numpy().astype(np.float64)
        total = float(sum(active_bytes(d, E, de, L, int(n)) for n in n_host))
        tps = C * L / (ms * 1e-3)
        gbs = total / (ms * 1e-3) / 1e9
        cls = 1.0 - float(n_host.mean()) / E
        line = {"metric": METRIC, "value": round(tps, 1), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": f"tls_sweep_{R}layers_d{d}_E{E}_de{de}_L{L}",
                           "point": "dense (every expert active)" if dense else f"tls {tls}",
                           "layers": R, "chunks_per_step": C, "teams": K,
                           "weights_gb": round(R * E * 2 * d * de * 2 / 1e9, 2),
                           "tls_measured": round(float(zeros.mean()) / (L * E), 4), "cls_measured": round(cls, 4),
                           "mean_n_active": round(float(n_host.mean()), 3)},
                "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                             "frac": round(gbs / peak, 4), "peak_kind": peak_kind,
                             "us_per_chunk": round(ms * 1e3 / C, 3)},
                "gpu_launches": 2 * args.steps, "clocks": clk.summary(), "gen_seconds": round(gen_s, 1)}
        if dense:
            dense_tps = tps
        else:
            line["speedup_vs_dense"] = round(tps / dense_tps, 3)
            line["speedup_bound"] = round(1.0 / max(1e-9, 1.0 - cls), 3)
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------- cross-chunk reuse
def run_dense_ffn(args):
    """The sweep's comparison point in a library: a dense FFN of the stacked model's shape (--replicas
    layers, default 32, of d = 4096 and E de = 32768 hidden units, 17.2 GB of bf16 weights) as plain cuBLAS
    bf16 GEMMs through torch, one chunk of L = 8 tokens at a time, 8 chunks per layer per step, as the sweep
    visits them: y = Swish(x W1^T) W2^T.  Random weights (their values do not change the time); HBM-bound
    like the sweep, so the line reports tokens/s and GB/s over the weight bytes."""
    import torch

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    R, d, H, L = args.replicas or 32, 4096, 128 * 256, 8
    per_layer = 8
    gen_t = torch.Generator(device=device).manual_seed(0)
    W1 = torch.randn((R, H, d), dtype=torch.bfloat16, device=device, generator=gen_t).mul_(d ** -0.5)
    W2 = torch.randn((R, d, H), dtype=torch.bfloat16, device=device, generator=gen_t).mul_(256 ** -0.5)
    x = torch.randn((R * per_layer, L, d), dtype=torch.bfloat16, device=device, generator=gen_t)
    y = torch.empty_like(x)
    s = torch.cuda.Stream(device)

    def step():
        for c in range(R * per_layer):
            l = c % R
            y[c] = torch.nn.functional.silu(x[c] @ W1[l].t()) @ W2[l].t()

    with torch.cuda.stream(s):
        step()
        s.synchronize()
        graph = torch.cuda.CUDAGraph()
        graph.capture_begin()
        step()
        graph.capture_end()
        for _ in range(args.warmup):
            graph.replay()
        s.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(0) as clocks:
            e0.record(s)
            for _ in range(args.steps):
                graph.replay()
            e1.record(s)
            e1.synchronize()
        del graph
    ms = e0.elapsed_time(e1) / args.steps
    chunks = R * per_layer
    bytes_step = chunks * (2 * H * d * 2 + L * d * 2 * 2)
    peak, peak_kind = measured_peaks()
    gbs = bytes_step / (ms * 1e-3) / 1e9
    line = {"metric": "dense FFN (cuBLAS bf16 through torch) tokens/s at chunk L=8, the stacked model's shape",
            "value": round(chunks * L / (ms * 1e-3), 1), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (random weights)",
            "config": {"workload": f"dense_ffn_layers{R}_d{d}_hidden{H}_L{L}", "chunks_per_step": chunks,
                       "l2": f"inputs larger than L2: {R * 2 * H * d * 2 / 1e9:.1f} GB of weights"},
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(gbs / peak, 4), "peak_kind": peak_kind, "traffic": None},
            "gpu_launches": 0, "library": "cuBLAS (torch.matmul) and a torch SiLU kernel", "clocks": clocks.summary()}
    print(json.dumps(line), flush=True)


def run_reuse(args):
    """Cross-chunk expert reuse on the per-chunk path (one chunk at a time on the whole GPU): the
    consecutive verification chunks of one sequence, as a drifting sequence of chunk bases (gen's
    make_sequence_chunks, --drift list).  For each drift: the mean reuse rate |U_k ∩ U_(k-1)| / |U_k|
    (blockffn_union_overlap on the device), and tokens/s with the experts' weights read evict-first
    (default) and evict-last (BFFN_FLAG_KEEP_EXPERTS_IN_L2), (a) one layer, steps back to back, and
    (b) the sequence through a stack of --replicas layers, step k visiting every layer before step k+1,
    as autoregressive decoding does.  One JSON line per drift and case."""
    import numpy as np
    import torch

    import chunk_sparse_moe_router_b200 as bffn
    import gen

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    w = gen.workload("decode")
    R = args.replicas or 16
    d, E, de, L = w.d, w.E, w.de, w.L
    n_steps = args.chunks or 256
    lays = [w.layer(r) for r in range(R)]
    dev = {k: [] for k in ("Wr", "br", "g", "W1", "W2")}
    for lay in lays:
        dev["Wr"].append(torch.from_numpy(lay.Wr).to(device))
        dev["br"].append(torch.from_numpy(lay.br).to(device))
        dev["g"].append(torch.from_numpy(lay.g).to(device))
        dev["W1"].append(torch.from_numpy(lay.W1.view(np.int16)).to(device))
        dev["W2"].append(torch.from_numpy(lay.W2.view(np.int16)).to(device))
    peak, peak_kind = measured_peaks()
    ws = bffn.new_workspace(L, d, E, de, device)
    ws_bytes = bffn.blockffn_workspace_size(L, d, E, de)
    s = torch.cuda.Stream(device)
    for drift in [float(v) for v in args.drift.split(",")]:
        for case, layers in (("one layer, steps back to back", 1), (f"{R} layers per step", R)):
            # x[k, l]: step k's chunk at layer l (each layer sees its own drifting sequence)
            xs = np.stack([gen.make_sequence_chunks(w.seed, lays[l], n_steps, L, w.noise, drift, stream=l)
                           for l in range(layers)], axis=1)
            x = torch.from_numpy(xs.view(np.int16)).to(device)
            y = torch.empty((n_steps, layers, L, d), dtype=torch.float32, device=device)
            idx = torch.full((n_steps, layers, E), -1, dtype=torch.int32, device=device)
            nact = torch.zeros((n_steps, layers), dtype=torch.int32, device=device)
            line_base = None
            for keep in (False, True):
                flags = bffn.BFFN_FLAG_KEEP_EXPERTS_IN_L2 if keep else 0

                def step():
                    for k in range(n_steps):
                        for l in range(layers):
                            rc = bffn.blockffn_chunk_forward_ex(
                                x[k, l].data_ptr(), L, d, dev["Wr"][l].data_ptr(), dev["g"][l].data_ptr(),
                                dev["W1"][l].data_ptr(), dev["W2"][l].data_ptr(), E, de, y[k, l].data_ptr(),
                                idx[k, l].data_ptr(), nact[k, l:].data_ptr(), dev["br"][l].data_ptr(), None, None,
                                None, flags, ws.data_ptr(), ws_bytes, s.cuda_stream)
                            if rc != 0:
                                raise bffn.BlockFFNError(rc, "blockffn_chunk_forward_ex")

                with torch.cuda.stream(s):
                    step()
                    s.synchronize()
                    graph = torch.cuda.CUDAGraph()
                    graph.capture_begin()
                    step()
                    graph.capture_end()
                    for _ in range(args.warmup):
                        graph.replay()
                    s.synchronize()
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(s)
                    for _ in range(args.steps):
                        graph.replay()
                    e1.record(s)
                    e1.synchronize()
                    if bffn.device_status(workspace=ws, stream=s.cuda_stream) != 0:
                        raise RuntimeError("device-side wait ran out")
                    del graph
                ms = e0.elapsed_time(e1) / args.steps
                calls = n_steps * layers
                # reuse rate of consecutive steps at each layer
                ov = torch.empty(((n_steps - 1) * layers,), dtype=torch.int32, device=device)
                ia = idx[:-1].reshape(-1, E).contiguous()
                ib = idx[1:].reshape(-1, E).contiguous()
                na = nact[:-1].reshape(-1).contiguous()
                nb = nact[1:].reshape(-1).contiguous()
                rc = bffn.blockffn_union_overlap(ia.data_ptr(), na.data_ptr(), ib.data_ptr(), nb.data_ptr(),
                                                 ov.numel(), E, ov.data_ptr(), s.cuda_stream)
                if rc != 0:
                    raise bffn.BlockFFNError(rc, "blockffn_union_overlap")
                s.synchronize()
                reuse = float((ov.float() / nb.float().clamp(min=1)).mean().item())
                n_host = nact.cpu().numpy()
                total = float(sum(active_bytes(d, E, de, L, int(v)) for v in n_host.reshape(-1)))
                tps = calls * L / (ms * 1e-3)
                line = {"metric": METRIC, "value": round(tps, 1), "unit": "tokens/s", "n_gpus": 1,
                        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
                        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                        "data": "synthetic",
                        "config": {"workload": "reuse_decode_d2048_E64_de256_L8", "case": case, "drift": drift,
                                   "steps_per_sequence": n_steps, "layers": layers,
                                   "keep_experts_in_l2": keep, "mean_n_active": round(float(n_host.mean()), 3),
                                   "reuse_rate": round(reuse, 4)},
                        "roofline": {"bound": "hbm", "achieved": round(total / (ms * 1e-3) / 1e9, 1), "peak": peak,
                                     "unit": "GB/s", "frac": round(total / (ms * 1e-3) / 1e9 / peak, 4),
                                     "peak_kind": peak_kind, "us_per_chunk": round(ms * 1e3 / calls, 3)},
                        "gpu_launches": calls * args.steps}
                if keep and line_base:
                    line["speedup_vs_evict_first"] = round(tps / line_base, 3)
                line_base = tps
                print(json.dumps(line), flush=True)


def run_fp8(args):
    """The batched decode step on fp8 (e4m3) expert weights (blockffn_quantize_fp8 once, then
    blockffn_chunk_forward_batch_fp8 per step) on the decode workload's inputs, next to the bf16 batched
    call on the same inputs.  Roofline: the step's active bytes with one byte per expert weight (plus the
    per-(expert, j) scales) over its CUDA-event time."""
    import copy

    import numpy as np
    import torch

    import chunk_sparse_moe_router_b200 as bffn
    import gen

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    w = gen.workload("decode")
    chunks = args.chunks or w.n_chunks
    layers, stack, x_host_np = build_inputs(w, 0, device, chunks)
    L, d, E, de, R = w.L, w.d, w.E, w.de, w.replicas
    x_dev = torch.from_numpy(x_host_np.view(np.int16)).to(device).view(torch.bfloat16)
    y = torch.empty((chunks, L, d), dtype=torch.float32, device=device)
    y16 = torch.empty_like(y)
    idx = torch.empty((chunks, E), dtype=torch.int32, device=device)
    nact = torch.empty((chunks,), dtype=torch.int32, device=device)
    q = bffn.quantize_fp8(stack["W1"].view(R * E, de, d), stack["W2"].view(R * E, d, de), R)
    ws = torch.zeros(bffn.blockffn_batch_fp8_workspace_size(chunks, L, d, E, de), dtype=torch.uint8, device=device)
    ws16 = torch.zeros(bffn.blockffn_batch_workspace_size(chunks, L, d, E, de, bffn.BFFN_FLAGS_SHARE(8)),
                       dtype=torch.uint8, device=device)
    s = torch.cuda.Stream(device)

    def step_fp8():
        bffn.chunk_forward_batch_fp8(x_dev, stack["Wr"], stack["g"], q, y, idx, nact, br=stack["br"], workspace=ws,
                                     stream=s.cuda_stream)

    def step_bf16():
        bffn.chunk_forward_batch(x_dev, stack["Wr"], stack["g"], stack["W1"], stack["W2"], y16, idx, nact,
                                 br=stack["br"], teams=8, workspace=ws16, stream=s.cuda_stream)

    def timed(step, clocks=False):
        with torch.cuda.stream(s):
            step()
            s.synchronize()
            graph = torch.cuda.CUDAGraph()
            graph.capture_begin()
            step()
            graph.capture_end()
            for _ in range(args.warmup):
                graph.replay()
            s.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with ClockSampler(0) as clk:
                e0.record(s)
                for _ in range(args.steps):
                    graph.replay()
                e1.record(s)
                e1.synchronize()
            del graph
        return e0.elapsed_time(e1) / args.steps, clk.summary()

    ms16, _ = timed(step_bf16)
    ms, clk = timed(step_fp8)
    n_host = nact.cpu().numpy()
    fixed = 4 * d * E + 8 * E + 2 * L * d + 4 * L * d
    bytes_fp8 = float(sum(fixed + int(n) * (2 * d * de + 8 * de) for n in n_host)) + 4 * R
    bytes_bf16 = float(sum(active_bytes(d, E, de, L, int(n)) for n in n_host))
    peak, peak_kind = measured_peaks()
    gbs = bytes_fp8 / (ms * 1e-3) / 1e9
    line = {"metric": METRIC + " (fp8 e4m3 expert weights)", "value": round(chunks * L / (ms * 1e-3), 1),
            "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8 e4m3 weights (power-of-two scales), f16 MMA, fp32 accumulate", "data": "synthetic",
            "config": {**w.describe(), "chunks_per_step": chunks, "mean_n_active": round(float(n_host.mean()), 3),
                       "l2": f"inputs larger than L2: {R} weight replicas, "
                             f"{R * E * 2 * d * de / 1e9:.2f} GB of fp8 expert weights"},
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(gbs / peak, 4), "peak_kind": peak_kind, "traffic": None,
                         "bytes_per_chunk": round(bytes_fp8 / chunks, 1), "us_per_chunk": round(ms * 1e3 / chunks, 3)},
            "bf16_same_inputs": {"ms_per_step": round(ms16, 4), "tokens_per_s": round(chunks * L / (ms16 * 1e-3), 1),
                                 "frac": round(bytes_bf16 / (ms16 * 1e-3) / 1e9 / peak, 4)},
            "speedup_vs_bf16": round(ms16 / ms, 3),
            "gpu_launches": (3 + 2 * ((chunks + 511) // 512)) * args.steps, "clocks": clk}
    if not args.no_cpu_baseline:
        import oracle
        lay0 = copy.copy(w.layer(0))
        q1, q2, s1, s2, t2 = oracle.quantize_fp8(lay0.W1, lay0.W2, 1)
        lay0.W1, lay0.W2 = oracle.dequantize_fp8(q1, q2, s1, s2, t2)
        line["cpu_baseline"] = cpu_baseline(w, lay0, x_host_np, args.cpu_seconds)
    print(json.dumps(line), flush=True)


def run_backward(args):
    """The layer's backward (blockffn_layer_backward) for --chunks chunks of 8 tokens (default 512: 4096
    tokens) at the decode layer's shape (d = 2048, E = 64, de = 256) with a random upstream gradient.
    Roofline: the contraction flops of the step over the P active (token, expert) pairs (5 products of
    2 P d de: U, Q, dW2, dW1, dX; the router's are 4 T d E) over its CUDA-event time, against the measured
    bf16 tensor peak; the MMAs issued are about twice that (fp32 operands as bf16 hi + lo pairs).  P is
    counted on the host from the same inputs (every pre-activation keeps a margin from zero)."""
    import numpy as np
    import torch

    import chunk_sparse_moe_router_b200 as bffn
    import gen

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    C, L, d, E, de = args.chunks or 512, 8, 2048, 64, 256
    T = C * L
    lay = gen.make_layer(0, d, E, de, beta=0.84, var_x=1.09)
    x_np = gen.make_chunks(0, lay, C, L, 0.3).reshape(T, d)
    dy_np = np.random.default_rng(1).standard_normal((T, d)).astype(np.float32)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    bf = lambda bits: t(bits.view(np.int16)).view(torch.bfloat16)
    x, W1, W2 = bf(x_np), bf(lay.W1), bf(lay.W2)
    Wr, br, g, dy = t(lay.Wr), t(lay.br), t(lay.g), t(dy_np)
    ws = torch.empty(bffn.blockffn_layer_backward_workspace_size(T, d, E, de), dtype=torch.uint8, device=device)
    s = torch.cuda.Stream(device)

    def step():
        bffn.layer_backward(x, Wr, g, W1, W2, dy, br=br, workspace=ws, stream=s.cuda_stream)

    with torch.cuda.stream(s):
        step()
        s.synchronize()
        graph = torch.cuda.CUDAGraph()
        graph.capture_begin()
        step()
        graph.capture_end()
        for _ in range(args.warmup):
            graph.replay()
        s.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(0) as clocks:
            e0.record(s)
            for _ in range(args.steps):
                graph.replay()
            e1.record(s)
            e1.synchronize()
        del graph
    ms = e0.elapsed_time(e1) / args.steps
    s_host = gen.bf16_bits_to_f32(x_np).astype(np.float64) @ lay.Wr.astype(np.float64) + lay.br
    P = int((s_host > 0).sum())
    flops = 5 * 2.0 * P * d * de + 4.0 * T * d * E
    peak, peak_kind = measured_peaks("bf16_tflops")
    tf = flops / (ms * 1e-3) / 1e12
    line = {"metric": "BlockFFN layer backward tokens/s and achieved TFLOP/s (over the active pairs)",
            "value": round(T / (ms * 1e-3), 1), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16 x and weights; fp32 dy and gradients (hi + lo bf16 pairs on warp MMAs)",
            "data": "synthetic",
            "config": {"workload": f"backward_T{T}_d{d}_E{E}_de{de}", "tokens": T, "active_pairs": P,
                       "tls": round(1.0 - P / (T * E), 4),
                       "l2": "inputs larger than L2 (x, dy, the weights and the pair rows: about "
                             f"{(T * d * 6 + E * d * de * 4 + P * (de * 16 + d * 4)) / 1e9:.2f} GB per step)"},
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(tf / peak, 4), "peak_kind": peak_kind, "traffic": None,
                         "flops_per_step": flops},
            "gpu_launches": 18 * args.steps, "clocks": clocks.summary()}
    if not args.no_cpu_baseline:
        import oracle
        w = lambda b: gen.bf16_bits_to_f32(b).astype(np.float64)
        W1f, W2f = w(lay.W1), w(lay.W2)
        n, t0 = 0, time.time()
        while time.time() - t0 < args.cpu_seconds and n < T:
            oracle.layer_backward(w(x_np[n:n + 1]), lay.Wr, lay.br, lay.g, W1f, W2f, dy_np[n:n + 1])
            n += 1
        dt = time.time() - t0
        line["cpu_baseline"] = {"value": round(n / dt, 3), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": f"{n} tokens, one at a time (dense fp64), {dt:.1f} s"}
    print(json.dumps(line), flush=True)


def run_cls_losses(args):
    """The CLS-aware losses and their backward through the router (blockffn_cls_losses): one step = the
    activation-locality and chunk-sparsification losses of a training batch of --chunks chunks of 8 tokens
    (default 4096: 32768 tokens, x 128 MiB, above the 126 MB L2) with dS, dWr, db and dx, at the decode
    layer's router shape (d = 2048, E = 64).  Roofline: the step's algorithmic bytes (x read once, Wr, dS
    and dx written once) over its CUDA-event time; the kernels' shares come from the ncu launch list.
    The oracle is timed beside it on a bounded sample of whole chunks."""
    import numpy as np
    import torch

    import chunk_sparse_moe_router_b200 as bffn
    import gen

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    C, L, d, E, alpha = args.chunks or 4096, 8, 2048, 64, 4.0
    T = C * L
    lay = gen.make_layer(0, d, E, 8, beta=1.04, var_x=1.09)
    x_np = gen.make_chunks(0, lay, C, L, 0.3).reshape(T, d)
    x = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16).to(device)
    Wr, br = torch.from_numpy(lay.Wr).to(device), torch.from_numpy(lay.br).to(device)
    f32 = dict(dtype=torch.float32, device=device)
    loss, dS, dWr, db, dx = (torch.empty(2, **f32), torch.empty(T, E, **f32), torch.empty(d, E, **f32),
                             torch.empty(E, **f32), torch.empty(T, d, **f32))
    ws = torch.empty(bffn.blockffn_cls_losses_workspace_size(C, L, d, E), dtype=torch.uint8, device=device)
    s = torch.cuda.Stream(device)

    def step():
        bffn.cls_losses(x, C, L, Wr, br, alpha, 1.0, 1.0, loss, dS, dWr, db, dx, workspace=ws,
                        stream=s.cuda_stream)

    with torch.cuda.stream(s):
        step()
        s.synchronize()
        graph = torch.cuda.CUDAGraph()  # one step per replay: no host work between steps
        graph.capture_begin()
        step()
        graph.capture_end()
        for _ in range(args.warmup):
            graph.replay()
        s.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(0) as clocks:
            e0.record(s)
            for _ in range(args.steps):
                graph.replay()
            e1.record(s)
            e1.synchronize()
        clk = clocks.summary()
        del graph
    ms = e0.elapsed_time(e1) / args.steps
    alg = T * d * 2 + d * E * 4 + E * 4 + T * E * 4 + d * E * 4 + E * 4 + T * d * 4 + 8
    peak, peak_kind = measured_peaks()
    gbs = alg / (ms * 1e-3) / 1e9
    line = {"metric": "CLS-aware losses + router backward tokens/s and achieved HBM GB/s over the step's I/O",
            "value": round(T / (ms * 1e-3), 1), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp32 (bf16 x; fp32 operands as bf16 hi+lo pairs on the tensor cores)",
            "data": "synthetic",
            "config": {"workload": f"cls_losses_C{C}_L{L}_d{d}_E{E}", "tokens": T, "alpha": alpha,
                       "l2": "inputs larger than L2 (x 128 MiB, dx 256 MiB written per step)"},
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(gbs / peak, 4), "peak_kind": peak_kind, "traffic": None,
                         "algorithmic_bytes_per_step": alg},
            "losses": [round(float(v), 6) for v in loss.cpu()],
            "gpu_launches": 6 * args.steps, "clocks": clk}
    if not args.no_cpu_baseline:
        import oracle
        n = 0
        t0 = time.time()
        while time.time() - t0 < args.cpu_seconds and n < C:
            m = min(64, C - n)
            oracle.cls_losses(x_np[n * L:(n + m) * L], m, L, lay.Wr, lay.br, alpha)
            n += m
        dt = time.time() - t0
        line["cpu_baseline"] = {"value": round(n * L / dt, 1), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": f"{n} chunks ({n * L} tokens) in groups of 64 chunks, {dt:.1f} s"}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------- CPU oracle
def cpu_baseline(w, lay0, x_host_np, seconds, y_gpu=None, n_gpu=None):
    """The fp64 dense oracle timed on this host's cores on a bounded sample of the workload (tokens
    of the chunks that use replica 0, in groups of up to 8).  Also checks that sample against the
    GPU's output when one is given."""
    import numpy as np

    import oracle

    cores = oracle.available_cores()
    L, d = w.L, w.d
    chunk_ids = list(range(0, x_host_np.shape[0], w.replicas))  # chunks that use replica 0
    toks = x_host_np[chunk_ids].reshape(len(chunk_ids) * L, d)
    group = min(L, 8)
    # warm up on one group, calibrate on two, then size the sample to about `seconds`
    oracle.tokens_forward_mt(toks[:group], lay0.Wr, lay0.br, lay0.g, lay0.W1, lay0.W2, cores)
    t0 = time.time()
    oracle.tokens_forward_mt(np.repeat(toks[:group], 2, axis=0), lay0.Wr, lay0.br, lay0.g, lay0.W1, lay0.W2, cores)
    t_group = (time.time() - t0) / 2
    n_groups = max(1, min(toks.shape[0] // group, int(seconds / max(t_group, 1e-6))))
    n_tok = n_groups * group
    t0 = time.time()
    y_ref = oracle.tokens_forward_mt(toks[:n_tok], lay0.Wr, lay0.br, lay0.g, lay0.W1, lay0.W2, cores)
    dt = time.time() - t0
    res = {"value": round(n_tok / dt, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
           "sample": f"{n_tok} tokens of weight replica 0's chunks "
                     f"(dense fp64: all {w.E} experts per token), {dt:.1f} s"}
    if y_gpu is not None:
        yg = y_gpu[chunk_ids].reshape(len(chunk_ids) * L, d)[:n_tok].cpu().numpy().astype(np.float64)
        bad = 0
        for a in range(0, n_tok, L):  # the tolerance's rms is taken per chunk
            yr, yc = y_ref[a:a + L], yg[a:a + L]
            bound = 2e-2 * np.abs(yr) + 1e-3 * np.sqrt(np.mean(yr ** 2))
            bad += int((np.abs(yc - yr) > bound).sum())
        res["parity_sample"] = {"y_elements_out_of_tolerance": bad, "elements": int(yg.size)}
    return res


def run_reference(args, w):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import numpy as np

    import gen
    import oracle

    lay = w.layer(0)
    L = w.L
    cores = oracle.available_cores()
    per_step_tokens = max(1, args.ref_chunks) * min(L, 8)  # decode: whole chunks; prefill: 8 tokens each
    x = gen.make_chunks(w.seed, lay, 1 if L > 8 else max(1, args.ref_chunks), L, w.noise, stream=0)
    xs = x.reshape(-1, w.d)[:per_step_tokens]
    oracle.tokens_forward_mt(xs[:min(L, 8)], lay.Wr, lay.br, lay.g, lay.W1, lay.W2, cores)  # warm-up
    t0 = time.time()
    for _ in range(args.steps):
        oracle.tokens_forward_mt(xs, lay.Wr, lay.br, lay.g, lay.W1, lay.W2, cores)
    dt = time.time() - t0
    value = args.steps * per_step_tokens / dt
    sample = (f"each step: {per_step_tokens} tokens of the workload, dense fp64 oracle "
              f"(all {w.E} experts per token)")
    out = {"metric": METRIC_PREFILL if L > DECODE_MAX_L else METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "impl": "reference",
           "config": {**w.describe(), "tokens_per_step": per_step_tokens},
           "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def _reference_line(args, metric, config, units_per_step, step, sample, cores):
    """Times `step` (one bounded sample of the workload through the oracle) --steps times after one warm-up
    call and prints the reference arm's JSON line (tokens/s)."""
    world = dist_env()[0]
    step()
    t0 = time.time()
    for _ in range(args.steps):
        step()
    dt = time.time() - t0
    value = args.steps * units_per_step / dt
    out = {"metric": metric, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
           "config": {**config, "tokens_per_step": units_per_step},
           "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_reference_workload(args):
    """The reference arm (the fp64 oracle on the host) for the workloads with their own runners: the
    CLS-aware losses, the fp8 decode layer (the oracle's forward on the dequantised weights) and the layer
    backward.  Rank 0 only; the same metric and config names as the GPU runner."""
    if dist_env()[1] != 0:
        return
    import copy

    import numpy as np

    import gen
    import oracle

    cores = oracle.available_cores()
    if args.workload == "cls_losses":
        C, L, d, E, alpha = args.chunks or 4096, 8, 2048, 64, 4.0
        lay = gen.make_layer(0, d, E, 8, beta=1.04, var_x=1.09)
        m = 64
        x_np = gen.make_chunks(0, lay, m, L, 0.3).reshape(m * L, d)
        _reference_line(args, "CLS-aware losses + router backward tokens/s and achieved HBM GB/s over the step's I/O",
                        {"workload": f"cls_losses_C{C}_L{L}_d{d}_E{E}", "tokens": C * L, "alpha": alpha}, m * L,
                        lambda: oracle.cls_losses(x_np, m, L, lay.Wr, lay.br, alpha),
                        f"each step: {m} chunks of {L} tokens, the fp64 oracle's losses and gradients (one core)", 1)
    elif args.workload == "fp8":
        w = gen.workload("decode")
        lay = copy.copy(w.layer(0))
        q1, q2, s1, s2, t2 = oracle.quantize_fp8(lay.W1, lay.W2, 1)
        lay.W1, lay.W2 = oracle.dequantize_fp8(q1, q2, s1, s2, t2)
        n = max(1, args.ref_chunks) * w.L
        xs = gen.make_chunks(w.seed, lay, max(1, args.ref_chunks), w.L, w.noise, stream=0).reshape(-1, w.d)[:n]
        _reference_line(args, METRIC + " (fp8 e4m3 expert weights)",
                        {**w.describe(), "chunks_per_step": args.chunks or w.n_chunks}, n,
                        lambda: oracle.tokens_forward_mt(xs, lay.Wr, lay.br, lay.g, lay.W1, lay.W2, cores),
                        f"each step: {n} tokens, dense fp64 oracle on the dequantised fp8 weights "
                        f"(all {w.E} experts per token)", cores)
    elif args.workload == "backward":
        C, L, d, E, de = args.chunks or 512, 8, 2048, 64, 256
        lay = gen.make_layer(0, d, E, de, beta=0.84, var_x=1.09)
        n = 4
        x_np = gen.make_chunks(0, lay, 1, L, 0.3).reshape(L, d)[:n]
        dy_np = np.random.default_rng(1).standard_normal((n, d)).astype(np.float32)
        wf = lambda b: gen.bf16_bits_to_f32(b).astype(np.float64)
        W1f, W2f, xf = wf(lay.W1), wf(lay.W2), wf(x_np)
        _reference_line(args, "BlockFFN layer backward tokens/s and achieved TFLOP/s (over the active pairs)",
                        {"workload": f"backward_T{C * L}_d{d}_E{E}_de{de}", "tokens": C * L}, n,
                        lambda: oracle.layer_backward(xf, lay.Wr, lay.br, lay.g, W1f, W2f, dy_np),
                        f"each step: {n} tokens, the fp64 oracle's backward (dense over the experts, one core)", 1)
    else:
        raise ValueError(args.workload)


def launch_local_ranks(n: int, argv: list[str]) -> int:
    """Run this script as n ranks on this node (one process per GPU, rendezvous on 127.0.0.1) when it
    was started without a launcher; returns the launcher's exit status."""
    import socket

    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        port = sock.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode",
                    choices=["decode", "tiny", "lsweep", "tls_sweep", "prefill", "reuse", "cls_losses", "fp8", "backward",
                             "dense_ffn"])
    ap.add_argument("--drift", default="0.0,0.9,0.97",
                    help="--workload reuse: drift of the chunk bases of a sequence (0: independent chunks)")
    ap.add_argument("--L", type=int, default=None, help="chunk length for --workload lsweep")
    ap.add_argument("--tls", type=float, default=None, help="token-level sparsity for --workload tls_sweep")
    ap.add_argument("--chunks", type=int, default=None, help="chunks per step (default: the workload's)")
    ap.add_argument("--tls-list", default="0.5,0.7,0.8,0.9,0.95",
                    help="--workload tls_sweep: the token-level sparsity points (a dense point is always added)")
    ap.add_argument("--replicas", type=int, default=None,
                    help="weight replicas (default: the workload's; keep their weights above the 126 MB L2)")
    ap.add_argument("--streams", type=int, default=8,
                    help="decode: independent chunks in flight at once (teams of SMs), each on 1/streams of them")
    ap.add_argument("--mode", choices=["batch", "streams"], default="batch",
                    help="decode chunks of up to 8 tokens: one batched call per step (default), or one call per "
                         "chunk on --streams streams")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-chunks", type=int, default=1)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(launch_local_ranks(args.gpus, sys.argv[1:]))
    if args.gpus != dist_env()[0]:
        ap.error(f"--gpus {args.gpus} but the launcher started {dist_env()[0]} ranks")

    import gen

    kw = {}
    if args.workload == "lsweep" and args.L:
        kw["L"] = args.L
    if args.workload == "tls_sweep" and args.tls:
        kw["tls"] = args.tls
    if args.replicas:
        kw["replicas"] = args.replicas
    if args.workload == "tls_sweep" and args.impl == "ours" and not args.tls:
        run_tls_sweep(args)
        return
    if args.impl == "reference" and args.workload in ("cls_losses", "fp8", "backward"):
        run_reference_workload(args)
        return
    if args.impl == "reference" and args.workload == "reuse":  # the reuse runs are the decode layer's forward
        run_reference(args, gen.workload("decode"))
        return
    if args.workload == "dense_ffn":
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the dense cuBLAS FFN is itself a comparison "
                              "point; its oracle is the decode layer's (--workload tls_sweep --impl reference)"}))
            return
        run_dense_ffn(args)
        return
    if args.workload == "reuse":
        run_reuse(args)
        return
    if args.workload == "cls_losses":
        run_cls_losses(args)
        return
    if args.workload == "fp8":
        run_fp8(args)
        return
    if args.workload == "backward":
        run_backward(args)
        return
    w = gen.workload(args.workload, **kw)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
