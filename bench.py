#!/usr/bin/env python
"""Benchmark of the routed-MoE decode with a streamed LFU expert cache.

Default workload (one "step" = one decode token through all 30 MoE layers):
  decode_stream  30 layers of the Gemma 4 26B-A4B MoE shape (d_model 2816,
                 128 experts, top-8, expert FFN 704, shared FFN 2112, 4-bit
                 group-64 experts, 8-bit router), batch 1, a 16-slot LFU cache
                 per layer in HBM, all 30 x 128 expert blobs (12.85 GB) in
                 pinned host memory, misses copied on a side stream while the
                 shared expert runs; router biased by a per-layer Zipf(s=1.1)
                 popularity so top-8 sets repeat; layer l+1's input is the
                 residual stream after layer l, RMS-normalised (serial
                 dependence).  Warm-up W tokens then K timed tokens from a cold
                 cache (defaults 16 + 240 = a 256-token sequence).
Other workloads (--workload): decode_resident (all experts in HBM, --batch
1/8/32), prefill (one 128-token chunk per layer, cold caches).

Prints one JSON line (rank 0).  Under torchrun every rank runs an independent
replica on its own GPU (the decode shards only across independent sequences);
time is the max over ranks.  `--impl reference` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE decode tokens/s (30 layers, top-8/128, 4-bit g64); HBM GB/s vs peak"
METRIC_PREFILL = "MoE prefill tokens/s (30 layers, 128-token chunks, top-8/128, 4-bit g64, cold 16-slot caches)"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=240)
    p.add_argument("--warmup", type=int, default=16)
    p.add_argument("--impl", default="b200", choices=["b200", "reference"])
    p.add_argument("--workload", default="decode_stream",
                   choices=["decode_stream", "decode_resident", "prefill", "sweep", "attn_decode"])
    p.add_argument("--sweep-tokens", type=int, default=4096)
    p.add_argument("--batch", type=int, default=1)
    p.add_argument("--slots", type=int, default=16)
    p.add_argument("--policy", choices=["lfu", "lru", "lfu_decay", "lfu_in_cache"], default="lfu",
                   help="slot-cache replacement rule of the streamed workloads (default lfu, the pages' rule)")
    p.add_argument("--decay-period", type=int, default=64, help="lfu_decay: halve the counts every N steps")
    p.add_argument("--store-file", default=None, metavar="DIR",
                   help="streamed workloads: write each layer's experts to DIR/layerNN.experts and read misses "
                        "from those files with positional reads (the file-backed store)")
    p.add_argument("--direct", action="store_true", help="--store-file: open the files with O_DIRECT")
    p.add_argument("--fill", choices=["direct", "copy"], default="copy",
                   help="streamed workloads with the pinned store: how one-token misses reach their slots -- "
                        "'copy': the host reads the plan and the copy engine copies them (default); "
                        "'direct': the one-launch layer kernel reads them from pinned host memory as it computes")
    p.add_argument("--lookahead", type=int, default=1, choices=[1, 2],
                   help="layers ahead the look-ahead may stage for: 2 = also the layer after next when the next "
                        "layer is predicted to miss nothing (measured: no gain, 178.6 vs 180.8 tokens/s)")
    p.add_argument("--prefetch", type=int, default=None, metavar="P",
                   help="decode_stream with --fill copy: stage up to P of the next layer's predicted misses "
                        "(look-ahead; 0 = off; default 1 for the one-token streamed decode from the pinned store)")
    p.add_argument("--zipf", type=float, default=None,
                   help="Zipf exponent of the router popularity bias (default 1.1; 0 = uniform router, "
                        "the default for decode_resident)")
    p.add_argument("--zipf-lambda", type=float, default=synth_default_lambda(),
                   help="strength of the Zipf popularity bias: bias_e = -lambda * s * ln(1 + rank_e); "
                        "calibrated so the chained 16-slot decode lands in the pages' 60-70%% hit-rate band")
    p.add_argument("--layers", type=int, default=30)
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu", action="store_true")
    p.add_argument("--profile", action="store_true", help="short run for ncu: no clocks, e2e or cpu legs")
    a = p.parse_args()
    if a.zipf is None:
        a.zipf = 0.0 if a.workload == "decode_resident" else 1.1
    if a.prefetch is None:
        a.prefetch = 1 if (a.workload == "decode_stream" and a.batch == 1 and not a.store_file
                           and a.fill == "copy") else 0
    if a.prefetch and (a.workload != "decode_stream" or a.batch != 1 or a.store_file or a.fill != "copy"):
        p.error("--prefetch needs the one-token decode_stream workload with the pinned host store and --fill copy")
    if not 0 <= a.prefetch <= 16:
        p.error("--prefetch takes 0..16 buffers")
    return a


# --------------------------------------------------------------- helpers
def synth_default_lambda():
    from expert_streaming_decode_b200 import synth
    return synth.ZIPF_LAMBDA


# sources of the one-token expert GEMV kernels whose DRAM traffic profiles/traffic.json records
TRAFFIC_SOURCES = ("ffn.cu", "ffn.cuh", "common.cuh", "decode_wl.cuh", "launch.cuh")


def csrc_sha256(files=TRAFFIC_SOURCES):
    """Hash of the kernel sources: DRAM traffic recorded under profiles/ is
    reported only for the kernel source it was measured on."""
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "expert_streaming_decode_b200", "csrc")
    for f in sorted(files):
        h.update(f.encode())
        h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()


def recorded_traffic(key, name="traffic.json", table="bytes_per_layer_token"):
    """DRAM bytes (read + write) of one kernel on one workload from one ncu
    capture (profiles/<name>): per layer-token for the expert GEMV kernels,
    per step for decode attention.  None when absent or taken on other kernel
    sources."""
    p = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(p):
        return None
    rec = json.load(open(p))
    if rec.get("source_sha256") != csrc_sha256(tuple(rec.get("sources", TRAFFIC_SOURCES))):
        return None
    return rec.get(table, {}).get(key)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        time.sleep(0.3)
        self.p.terminate()
        try:
            self.p.wait(5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.seek(0)
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.f.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.f.name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.local_world = int(os.environ.get("LOCAL_WORLD_SIZE", "1"))
        self.pg = None

    def init(self, backend):
        if self.world > 1:
            import datetime

            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        import torch
        t = torch.tensor([v], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def sum(self, v: float) -> float:
        if not self.pg:
            return v
        import torch
        t = torch.tensor([v], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
        self.pg.all_reduce(t, op=self.pg.ReduceOp.SUM)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ------------------------------------------------------- the host store
def mem_available() -> int:
    """Bytes the kernel reports as available for new allocations."""
    with open("/proc/meminfo") as f:
        for line in f:
            if line.startswith("MemAvailable:"):
                return int(line.split()[1]) * 1024
    return 0


class HostStore:
    """Every routed expert of every layer in host memory, [L][E][stride] uint8.

    One process per GPU on a node: the local ranks share ONE copy, a POSIX
    shared-memory segment that local rank 0 creates and fills and the others
    map; each rank then page-locks the mapping for its own GPU, so eight
    replicas hold one 12.85 GB store instead of eight.  A single process uses
    ordinary pinned memory.  Both refuse up front, with the numbers, when the
    host cannot hold the store (rather than failing half-way through pinning).
    `pin` False keeps the memory pageable (CPU tests)."""

    SHM_DIR = "/dev/shm"

    def __init__(self, shape, fill, dist, pin=True, tag="moe_store", avail=None):
        import mmap

        import torch
        self.shape, self.nbytes = tuple(shape), int(np.prod(shape))
        self._mm, self._path, self.registered = None, None, False
        avail = mem_available() if avail is None else avail
        if dist.local_world <= 1:
            if self.nbytes > 0.9 * avail:
                raise RuntimeError(f"host store of {self.nbytes / 1e9:.2f} GB does not fit: "
                                   f"{avail / 1e9:.2f} GB available")
            self.tensor = torch.empty(self.shape, dtype=torch.uint8, pin_memory=pin)
            fill(self.tensor.numpy())
            self.shared = False
            return
        st = os.statvfs(self.SHM_DIR)
        shm_free = st.f_bavail * st.f_frsize
        if self.nbytes > shm_free or self.nbytes > 0.9 * avail:
            raise RuntimeError(f"{dist.local_world} local ranks share one host store of {self.nbytes / 1e9:.2f} GB, "
                               f"but {self.SHM_DIR} has {shm_free / 1e9:.2f} GB free and the host "
                               f"{avail / 1e9:.2f} GB available")
        self._path = os.path.join(self.SHM_DIR, f"{tag}_{os.environ.get('MASTER_PORT', '0')}")
        if dist.local == 0:
            try:
                fd = os.open(self._path, os.O_CREAT | os.O_EXCL | os.O_RDWR, 0o600)
            except FileExistsError:
                # left behind by an earlier run on this port that did not finish
                os.unlink(self._path)
                fd = os.open(self._path, os.O_CREAT | os.O_EXCL | os.O_RDWR, 0o600)
            try:
                os.ftruncate(fd, self.nbytes)
                self._mm = mmap.mmap(fd, self.nbytes)
            finally:
                os.close(fd)
            fill(np.frombuffer(self._mm, dtype=np.uint8).reshape(self.shape))
        dist.barrier()
        if dist.local != 0:
            fd = os.open(self._path, os.O_RDWR)
            try:
                self._mm = mmap.mmap(fd, self.nbytes)
            finally:
                os.close(fd)
        dist.barrier()
        if dist.local == 0:
            os.unlink(self._path)  # every rank holds a mapping; the name is no longer needed
        self._path = None
        self.tensor = torch.from_numpy(np.frombuffer(self._mm, dtype=np.uint8).reshape(self.shape))
        self.shared = True
        if pin:
            # page-locked for this rank's GPU; mapped, so kernels can read it
            rc = torch.cuda.cudart().cudaHostRegister(self.tensor.data_ptr(), self.nbytes, 3)
            if int(rc) != 0:
                raise RuntimeError(f"cudaHostRegister of the shared host store failed ({int(rc)})")
            self.registered = True

    def close(self):
        if self.registered:
            import torch
            torch.cuda.cudart().cudaHostUnregister(self.tensor.data_ptr())
            self.registered = False
        self.tensor = None
        if self._mm is not None:
            try:
                self._mm.close()
            except BufferError:
                pass  # views still alive; the mapping goes with the process
            self._mm = None


# ------------------------------------------------------------- the model
class Model:
    """30 MoE layers of synthetic weights: routers, shared experts and the
    routed expert blobs, either streamed (pinned host store + HBM slot
    caches) or resident in HBM."""

    def __init__(self, args, dims, max_tokens, streaming, store=None, dist=None):
        import torch

        from expert_streaming_decode_b200 import moe, synth
        self.moe, self.synth, self.torch = moe, synth, torch
        self.d, self.L, self.S = dims, args.layers, args.slots
        self.streaming = streaming
        self.nb = synth.blob_bytes(dims.D, dims.F)
        self.stride = (self.nb + 255) // 256 * 256
        self.ctx = moe.Ctx.from_dims(dims, max_tokens=max_tokens, S=args.slots)
        dev = torch.device("cuda")
        self.wq, self.ws, self.bias, self.shared = [], [], [], []
        for l in range(self.L):
            wq, ws = synth.router_weights(args.seed, l, dims.E, dims.D)
            self.wq.append(torch.from_numpy(wq).to(dev))
            self.ws.append(torch.from_numpy(ws.view(np.int16)).to(dev))
            b = synth.zipf_bias(args.seed, l, dims.E, s=args.zipf, lam=args.zipf_lambda) if args.zipf > 0 else None
            self.bias.append(None if b is None else torch.from_numpy(b).to(dev))
            self.shared.append(torch.from_numpy(synth.expert_blob(args.seed, l, 0, dims.D, dims.FS, shared=True)).to(dev))
        t0 = time.time()
        self.host_store = None
        if store is None:
            sd = synth.Dims(**{**dims.as_dict(), "L": self.L})

            def fill(view):
                synth.fill_store(view[:, :, :self.nb], args.seed, sd)
            if streaming:
                self.host_store = HostStore((self.L, dims.E, self.stride), fill, dist or Dist())
                store = self.host_store.tensor
            else:
                store = torch.empty((self.L, dims.E, self.stride), dtype=torch.uint8)
                fill(store.numpy())
        self.gen_s = time.time() - t0
        if streaming:
            self.store = store
            self.slots = [torch.empty((self.S, self.stride), dtype=torch.uint8, device=dev) for _ in range(self.L)]
            self.state = [torch.empty(self.ctx.state_words(), dtype=torch.int32, device=dev) for _ in range(self.L)]
            pol = {"lfu": moe.MOE_POLICY_LFU, "lru": moe.MOE_POLICY_LRU, "lfu_decay": moe.MOE_POLICY_LFU_DECAY,
                   "lfu_in_cache": moe.MOE_POLICY_LFU_IN_CACHE}[getattr(args, "policy", "lfu")]
            per = getattr(args, "decay_period", 0) if pol == moe.MOE_POLICY_LFU_DECAY else 0
            self.fds, self.files = [], []
            if getattr(args, "store_file", None):
                # one file per layer, experts at a 4 KB-aligned stride (O_DIRECT-compatible)
                fstride = (self.nb + 4095) // 4096 * 4096
                os.makedirs(args.store_file, exist_ok=True)
                view = store.numpy()
                pad = b"\0" * (fstride - self.nb)
                for l in range(self.L):
                    path = os.path.join(args.store_file, f"layer{l:02d}.experts")
                    with open(path, "wb") as f:
                        for e in range(dims.E):
                            f.write(view[l, e, :self.nb].tobytes())
                            f.write(pad)
                    self.files.append(path)
                    flags = os.O_RDONLY | (os.O_DIRECT if args.direct else 0)
                    self.fds.append(os.open(path, flags))
                self.caches = [moe.slot_cache(self.slots[l], self.stride, self.state[l], None, fstride,
                                              policy=pol, decay_period=per, store_fd=self.fds[l])
                               for l in range(self.L)]
            else:
                self.caches = [moe.slot_cache(self.slots[l], self.stride, self.state[l], store[l], self.stride,
                                              policy=pol, decay_period=per,
                                              direct=getattr(args, "fill", "copy") == "direct")
                               for l in range(self.L)]
            self.W = [moe.layer_weights(self.wq[l], self.ws[l], self.shared[l]) for l in range(self.L)]
            self.nexts = None
            self.lookahead = bool(getattr(args, "prefetch", 0))
            if getattr(args, "prefetch", 0) > 0:
                # layer l stages layer l+1's predicted misses; the last layer has
                # no successor within the token
                # (and, with --lookahead 2, layer l+2's when layer l+1 is
                # predicted to miss nothing)
                moe.prefetch_configure(self.ctx, args.prefetch)
                deep = getattr(args, "lookahead", 1) >= 2
                after = [moe.next_layer(self.W[l + 2], self.caches[l + 2], self.bias[l + 2])
                         if deep and l + 2 < self.L else None for l in range(self.L)]
                self.nexts = [moe.next_layer(self.W[l + 1], self.caches[l + 1], self.bias[l + 1], after=after[l])
                              for l in range(self.L - 1)] + [None]
        else:
            self.lookahead = False
            self.experts = store.to(dev)
            del store
            self.caches = [None] * self.L
            self.W = [moe.layer_weights(self.wq[l], self.ws[l], self.shared[l], self.experts[l], self.stride)
                      for l in range(self.L)]
            self.nexts = None

    def close_files(self):
        """Closes and deletes the expert files this run wrote (--store-file)."""
        for fd in getattr(self, "fds", []):
            os.close(fd)
        for path in getattr(self, "files", []):
            os.remove(path)
        self.fds, self.files = [], []

    def reset(self):
        if self.streaming:
            for c in self.caches:
                self.moe.cache_reset(self.ctx, c)

    def token_bytes_hbm(self, distinct_routed: float):
        """Algorithmic HBM bytes of one token-layer: weights streamed by the
        kernels plus activations (x in, h out/in, y out)."""
        d, s = self.d, self.synth
        gu = distinct_routed * (s.blob_bytes(d.D, d.F) - self._sec1(d.F)) + (s.blob_bytes(d.D, d.FS) - self._sec1(d.FS))
        dn = distinct_routed * self._sec1(d.F) + self._sec1(d.FS)
        router = d.E * d.D + d.E * d.D // 64 * 2
        return gu, dn, router

    def _sec1(self, F):
        ks = self.synth.down_ks(F)
        return (self.d.D // 32) * (F // ks) * 18 * ks


def moe_prefetch_stats(model):
    """(issued, used) look-ahead bytes so far; zeros when prefetch is off."""
    return model.moe.prefetch_stats(model.ctx) if model.lookahead else (0, 0)


def decode_token(model, x0, r, x, y, T, tok, tr=None, trace_acc=None, on_layer=None, ids=None, gate_w=None):
    """One decode step: T tokens through every layer (layer l+1 reads the
    residual stream after layer l, RMS-normalised).  on_layer(l, x_l, y, r),
    if given, runs after layer l's call and before the residual step (tests
    use it to read each layer's input and output); ids / gate_w receive the
    layer's routing when given."""
    moe, d, ctx = model.moe, model.d, model.ctx
    st = model.torch.cuda.current_stream()  # once per token: the library calls all go to it
    moe.bf16_to_f32(ctx, x0, r, T * d.D, stream=st)
    cur = x0
    for l in range(model.L):
        if model.nexts is not None and T == 1:
            moe.layer_forward_next(ctx, model.W[l], model.caches[l], cur, T, tok, model.bias[l], y, model.nexts[l],
                                   ids=ids, gate_w=gate_w, trace=tr, stream=st)
        else:
            moe.layer_forward(ctx, model.W[l], model.caches[l], cur, T, tok, model.bias[l], y, ids=ids,
                              gate_w=gate_w, trace=tr, stream=st)
        if tr is not None:
            res = tr.c
            trace_acc["misses"] += res.n_misses
            trace_acc["distinct"] += res.n_distinct
            trace_acc["h2d"] += int(res.h2d_bytes)
            if T == 1:
                # expert repeats across consecutive tokens of this layer
                sel = set(int(e) for e in tr.arrays["expert"][:res.n_distinct])
                hist = trace_acc.setdefault("hist", {}).setdefault(l, [])
                if len(hist) == 2:
                    trace_acc["rep_n"] = trace_acc.get("rep_n", 0) + len(sel)
                    trace_acc["rep1"] = trace_acc.get("rep1", 0) + len(sel & hist[-1])
                    trace_acc["rep2"] = trace_acc.get("rep2", 0) + len(sel & (hist[-1] | hist[-2]))
                hist.append(sel)
                del hist[:-2]
        if on_layer is not None:
            on_layer(l, cur, y, r)
        if l + 1 < model.L:
            moe.residual_rmsnorm(ctx, r, y, x, T, stream=st)
            cur = x


class Runner:
    """Runs decode steps; resident workloads replay a CUDA graph of one step
    (kernels chained with programmatic dependent launch), streamed ones call
    the library directly (each layer waits for its cache plan on the host)."""

    def __init__(self, model, T, graph):
        torch = model.torch
        self.m, self.T = model, T
        d = model.d
        self.x_in = torch.empty((T, d.D), dtype=torch.int16, device="cuda")
        self.x = torch.empty((T, d.D), dtype=torch.int16, device="cuda")
        self.r = torch.empty((T, d.D), dtype=torch.float32, device="cuda")
        self.y = torch.empty((T, d.D), dtype=torch.float32, device="cuda")
        self.graph = None
        self.launches_per_step = None
        self.cold_each_step = False
        if graph:
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s):  # warm-up outside capture
                decode_token(model, self.x_in, self.r, self.x, self.y, T, 0)
            torch.cuda.current_stream().wait_stream(s)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            l0 = model.ctx.launches
            with torch.cuda.graph(g):
                decode_token(model, self.x_in, self.r, self.x, self.y, T, 0)
            self.launches_per_step = model.ctx.launches - l0
            self.graph = g

    def run(self, x_src, steps, start_tok, trace_acc=None, host_io=None):
        """x_src: [n, T, D] device tensor of first-layer inputs (or None with
        host_io = (x_host_pinned, y_host_pinned))."""
        m, T = self.m, self.T
        tr = m.moe.Trace(m.d.E) if trace_acc is not None else None
        launches = 0
        for i in range(steps):
            tok = start_tok + i
            if self.cold_each_step:
                m.reset()  # a prefill chunk starts from cold caches
            if host_io is not None:
                xh, yh = host_io
                src = xh[tok % xh.shape[0]]
            else:
                src = x_src[tok % x_src.shape[0]]
            if self.graph is not None:
                self.x_in.copy_(src, non_blocking=True)
                self.graph.replay()
                launches += self.launches_per_step
            else:
                l0 = m.ctx.launches
                x0 = src.to("cuda", non_blocking=True) if host_io is not None else src
                decode_token(m, x0, self.r, self.x, self.y, T, tok, tr, trace_acc)
                launches += m.ctx.launches - l0
            if host_io is not None:
                host_io[1][tok % host_io[1].shape[0]].copy_(self.y, non_blocking=True)
        return launches


def timed(dist, model, fn):
    """Times fn() on the device between two events on the current stream,
    with a barrier and a synchronize on both sides; max over ranks."""
    torch = model.torch
    torch.cuda.synchronize()
    dist.barrier()
    st = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    out = fn()
    b.record(st)
    torch.cuda.synchronize()
    model.ctx.sync()
    dist.barrier()
    return dist.max(a.elapsed_time(b)), out


def file_read_peak_gbs(paths, chunk, direct, total=512 << 20, threads=4):
    """Positional-read bandwidth of the expert files: `total` bytes in `chunk`
    reads spread over the files, `threads` reads in flight (page-aligned
    buffers, so O_DIRECT descriptors work)."""
    import mmap
    import threading
    fds = [os.open(p, os.O_RDONLY | (os.O_DIRECT if direct else 0)) for p in paths]
    sizes = [os.fstat(fd).st_size for fd in fds]
    jobs = []
    while len(jobs) * chunk < total:
        k = len(jobs)
        f, o = k % len(fds), (k // len(fds)) * chunk
        if o + chunk > sizes[f]:
            break
        jobs.append((fds[f], o))
    lock = threading.Lock()

    def worker():
        buf = mmap.mmap(-1, chunk)
        while True:
            with lock:
                if not jobs:
                    return
                fd, o = jobs.pop()
            os.preadv(fd, [buf], o)
    n = len(jobs)
    t0 = time.time()
    ts = [threading.Thread(target=worker) for _ in range(threads)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    dt = time.time() - t0
    for fd in fds:
        os.close(fd)
    return n * chunk / dt / 1e9


def h2d_peak_gbs(torch):
    n = 256 << 20
    src = torch.empty(n, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(n, dtype=torch.uint8, device="cuda")
    best = 0.0
    for _ in range(6):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dst.copy_(src, non_blocking=True)
        b.record()
        torch.cuda.synchronize()
        best = max(best, n / (a.elapsed_time(b) * 1e-3) / 1e9)
    return best


# ------------------------------------------------------ CPU oracle timing
class OracleDecoder:
    """The CPU oracle running the same decode (router, LFU plan, expert FFNs,
    combine, and the harness residual/RMS step), one (token, layer) at a time;
    expert blobs regenerated on demand from the seeded generator."""

    def __init__(self, args, dims, first_token=0, blob_cache=600):
        import oracle

        from expert_streaming_decode_b200 import synth
        self.O, self.synth, self.d, self.args = oracle.get(), synth, dims, args
        self.blob_cache = blob_cache
        self.L = args.layers
        self.routers = [synth.router_weights(args.seed, l, dims.E, dims.D) for l in range(self.L)]
        self.bias = [synth.zipf_bias(args.seed, l, dims.E, s=args.zipf, lam=args.zipf_lambda) if args.zipf > 0
                     else None for l in range(self.L)]
        self.shared = {}
        self.blobs = {}
        pol = {"lfu": oracle.POLICY_LFU, "lru": oracle.POLICY_LRU, "lfu_decay": oracle.POLICY_LFU_DECAY,
               "lfu_in_cache": oracle.POLICY_LFU_IN_CACHE}[getattr(args, "policy", "lfu")]
        per = getattr(args, "decay_period", 0) if pol == oracle.POLICY_LFU_DECAY else 0
        self.lfu = [oracle.LfuState(dims.E, args.slots, pol, per) for _ in range(self.L)]
        self.tok, self.layer = first_token, 0
        self.x = synth.hidden(args.seed, first_token, 0, dims.D)
        self.r = synth.bf16_bits_to_f32(self.x).astype(np.float64)

    def _blob(self, l, e):
        k = (l, e)
        if k not in self.blobs:
            if len(self.blobs) > self.blob_cache:
                self.blobs.clear()
            self.blobs[k] = self.synth.expert_blob(self.args.seed, l, e, self.d.D, self.d.F)
        return self.blobs[k]

    def step(self):
        """One (token, layer)."""
        d, l = self.d, self.layer
        if l not in self.shared:
            self.shared[l] = self.synth.expert_blob(self.args.seed, l, 0, d.D, d.FS, shared=True)
        wq, ws = self.routers[l]

        class Lazy:
            def __getitem__(s, e):
                return self._blob(l, e)

        lg = self.O.router_logits(self.x, wq, ws, self.bias[l], d.E, d.D, d.G)
        ids = self.O.topk(lg, d.K)
        self.O.lfu_plan(self.lfu[l], ids[None], self.tok)
        blobs = Lazy()
        _, _, _, y = self.O.moe_token(d.as_dict(), self.x, wq, ws, self.bias[l], self.shared[l],
                                      [blobs[e] if e in ids else np.zeros(1, np.uint8) for e in range(d.E)])
        self.r, self.x = self.O.residual_rmsnorm(self.r, y)
        self.layer += 1
        if self.layer == self.L:
            self.layer = 0
            self.tok += 1
            self.x = self.synth.hidden(self.args.seed, self.tok, 0, d.D)
            self.r = self.synth.bf16_bits_to_f32(self.x).astype(np.float64)


def _oracle_worker(args, dims, budget_s, first_token):
    """One host core: the oracle's decode from `first_token` for budget_s."""
    dec = OracleDecoder(args, dims, first_token=first_token, blob_cache=64)
    t0 = time.perf_counter()
    n = 0
    while True:
        dec.step()
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 4 * args.layers:
            return n, el


def cpu_baseline(args, dims, budget_s=20.0, procs=None):
    """The oracle as it stands, on the host's cores: independent decode
    sequences (one per process, each starting at its own token) run side by
    side for about budget_s; throughput = all (token, layer) steps / the
    longest worker's time.  Processes are spawned, never forked from a
    process that has used the GPU."""
    import concurrent.futures as cf
    import multiprocessing as mp
    procs = procs or max(1, min(os.cpu_count() or 1, 32))
    if procs == 1:
        n, el = _oracle_worker(args, dims, budget_s, 0)
        res = [(n, el)]
    else:
        with cf.ProcessPoolExecutor(procs, mp_context=mp.get_context("spawn")) as ex:
            res = list(ex.map(_oracle_worker, [args] * procs, [dims] * procs, [budget_s] * procs,
                              [1000 * i for i in range(procs)]))
    n = sum(r[0] for r in res)
    el = max(r[1] for r in res)
    toks = n / args.layers
    return {"value": toks / el, "unit": "tokens/s", "cores": procs, "kind": "oracle",
            "sample": f"{procs} independent decode_stream sequences side by side, {n} (token, layer) steps "
                      f"({toks:.2f} tokens) in {el:.1f} s; plain C oracle (fp64), one process per core"}


def run_reference(args, dims, dist):
    if dist.rank != 0:
        return 0
    dec = OracleDecoder(args, dims)
    for _ in range(args.warmup):
        dec.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        dec.step()
    el = time.perf_counter() - t0
    toks = args.steps / args.layers
    v = toks / el
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "layers": args.layers, "batch": 1, "slots": args.slots,
                       "zipf_s": args.zipf, "step": "one (token, layer) of the decode sequence"},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": f"{args.steps} (token, layer) steps after {args.warmup} warm-up steps"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------- cache sweep
def run_sweep(args, dims, dist):
    """Cache sweep: for every (slots, Zipf s) the router + LFU plan run over
    --sweep-tokens decode tokens x 30 layers (seeded generator states for every
    (token, layer)), giving hit rate and H2D bytes/token; tokens/s comes from a
    short streamed decode (64 tokens after 16 warm-up) at the same point."""
    import torch

    from expert_streaming_decode_b200 import moe, synth
    d = dims
    nb = synth.blob_bytes(d.D, d.F)
    results = []
    routers = [synth.router_weights(args.seed, l, d.E, d.D) for l in range(args.layers)]
    wq = [torch.from_numpy(r[0]).cuda() for r in routers]
    ws = [torch.from_numpy(r[1].view(np.int16)).cuda() for r in routers]
    Tn = args.sweep_tokens
    t0 = time.time()
    xs_all = torch.empty((Tn, args.layers, d.D), dtype=torch.int16, device="cuda")
    for tok in range(Tn):
        blk = np.stack([synth.hidden(args.seed, tok, l, d.D) for l in range(args.layers)])
        xs_all[tok].copy_(torch.from_numpy(blk.view(np.int16)))
    gen_s = time.time() - t0
    def plan_point(S, zs, policy=moe.MOE_POLICY_LFU, period=0):
        """Router + cache plan over Tn tokens x all layers: hit rate and H2D bytes per token."""
        ctx = moe.Ctx.from_dims(d, max_tokens=1, S=S)
        # independent states per (token, layer): the unchained bias strength
        bias = [torch.from_numpy(synth.zipf_bias(args.seed, l, d.E, s=zs, lam=synth.ZIPF_LAMBDA_UNCHAINED)).cuda()
                for l in range(args.layers)]
        states = [torch.empty(ctx.state_words(), dtype=torch.int32, device="cuda") for _ in range(args.layers)]
        slots = torch.empty((S, 256), dtype=torch.uint8, device="cuda")  # plan only: never read
        caches = []
        for st in states:
            c = moe.slot_cache(slots, (nb + 255) // 256 * 256, st, policy=policy, decay_period=period)
            moe.cache_reset(ctx, c)
            caches.append(c)
        ids = torch.empty((1, d.K), dtype=torch.int32, device="cuda")
        gw = torch.empty((1, d.K), dtype=torch.float32, device="cuda")
        ps = torch.empty((1, d.K), dtype=torch.int32, device="cuda")
        tr = moe.Trace(d.E)
        hits = misses = 0
        t0 = time.time()
        for tok in range(Tn):
            for l in range(args.layers):
                moe.router_topk(ctx, xs_all[tok, l:l + 1], wq[l], ws[l], bias[l], 1, ids, gw)
                moe.cache_plan(ctx, caches[l], ids, 1, tok, ps, tr)
                r = tr.result()
                misses += r["misses"]
                hits += r["n_distinct"] - r["misses"]
        ctx.sync()
        ctx.close()
        return {"slots": S, "zipf_s": zs, "hit_rate": hits / max(1, hits + misses),
                "h2d_bytes_per_token": misses * nb / Tn, "plan_seconds": time.time() - t0}

    for S in (8, 16, 32, 64):
        for zs in (0.8, 1.1, 1.4):
            results.append(plan_point(S, zs))
    # replacement-rule variants at Zipf 1.1 (hit rate and H2D bytes; tokens/s follows the bytes)
    policies = []
    for name, pol, per in (("lru", moe.MOE_POLICY_LRU, 0), ("lfu_decay_64", moe.MOE_POLICY_LFU_DECAY, 64),
                           ("lfu_in_cache", moe.MOE_POLICY_LFU_IN_CACHE, 0)):
        for S in (8, 16, 32):
            policies.append({"policy": name, **plan_point(S, 1.1, pol, per)})
    # tokens/s at each point from a short streamed decode (one store for all)
    store = None
    for res in results:
        a2 = argparse.Namespace(**{**vars(args), "slots": res["slots"], "zipf": res["zipf_s"]})
        model = Model(a2, synth.Dims(L=args.layers, S=res["slots"]), max_tokens=1, streaming=True, store=store)
        store = model.store
        xs = np.stack([synth.hidden_batch(args.seed + 17, [i], 0, d.D) for i in range(80)])
        x_dev = torch.from_numpy(xs.view(np.int16)).cuda()
        runner = Runner(model, 1, graph=False)
        model.reset()
        runner.run(x_dev, 16, 0)
        ms, _ = timed(dist, model, lambda: runner.run(x_dev, 64, 16))
        res["tokens_per_s"] = 64 / (ms * 1e-3)
        model.ctx.close()
        del model
        torch.cuda.empty_cache()
    if dist.rank == 0:
        base = next(r for r in results if r["slots"] == 16 and abs(r["zipf_s"] - 1.1) < 1e-9)
        line = {"metric": "MoE decode cache sweep: hit rate, H2D bytes/token, tokens/s (30 layers, 4-bit g64)",
                "value": base["tokens_per_s"], "unit": "tokens/s", "n_gpus": dist.world, "steps": 64, "warmup": 16,
                "ms_per_step": 1e3 / base["tokens_per_s"], "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None,
                "dtype": "int4 weights x 16-bit fixed-point activations (dp4a), fp32 accumulation",
                "data": "synthetic",
                "config": {"workload": "sweep", "layers": args.layers, "sweep_tokens": Tn,
                           "value_point": "slots 16, zipf 1.1, LFU", "hidden_state_generation_s": gen_s,
                           "hit_rate_inputs": "independent hidden states per (token, layer), bias strength "
                                              f"{synth.ZIPF_LAMBDA_UNCHAINED}",
                           "tokens_per_s_inputs": "chained decode (residual stream), bias strength "
                                                  f"{args.zipf_lambda}"},
                "sweep": results, "policies": policies}
        print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------ decode attention
METRIC_ATTN = "decode attention tokens/s (30 layers: 25 sliding-window rings + 5 full, 4K context, fp16 KV)"


def _attn_layers(A):
    """(capacity, n_tokens) per layer: five sliding-window layers, then one
    full-attention layer, repeated; the context is full (steady decode)."""
    out = []
    for l in range(A.sliding + A.full):
        full = l % 6 == 5
        out.append((A.context if full else A.window, A.context))
    return out


def _attn_bytes(A, cap, n):
    """Algorithmic bytes of one launch: the attended K and V rows, q, o."""
    L = min(cap, n)
    return 2 * L * A.Hkv * A.hd * 2 + A.Hq * A.hd * 2 + A.Hq * A.hd * 4


def attn_cpu_baseline(A, seed, budget_s=20.0):
    """The oracle on a bounded sample: one sliding and one full layer for as
    many tokens as fit the budget, scaled to the 30-layer mix."""
    import oracle
    from expert_streaming_decode_b200 import synth
    O = oracle.get()
    layers = _attn_layers(A)
    cs = next(c for c in layers if c[0] == A.window)
    cf = next(c for c in layers if c[0] == A.context)
    ks, vs = synth.attn_kv(seed, 0, A.Hkv, cs[0], A.hd)
    kf, vf = synth.attn_kv(seed, 5, A.Hkv, cf[0], A.hd)
    ts = tf = 0.0
    n = 0
    t_start = time.perf_counter()
    while n < 1 or (time.perf_counter() - t_start < budget_s and n < 50):
        q = synth.attn_query(seed, n, 0, A.Hq, A.hd)
        t0 = time.perf_counter()
        O.attn_decode(q, ks, vs, cs[0], cs[1], 1.0 / math.sqrt(A.hd))
        t1 = time.perf_counter()
        O.attn_decode(q, kf, vf, cf[0], cf[1], 1.0 / math.sqrt(A.hd))
        t2 = time.perf_counter()
        ts += t1 - t0
        tf += t2 - t1
        n += 1
    per_tok = (A.sliding * ts + A.full * tf) / n
    return {"value": 1.0 / per_tok, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} tokens of one sliding-window and one full layer, scaled to 25 + 5 layers; "
                      f"single-threaded C oracle (fp64), {ts + tf:.1f} s"}


def run_reference_attn(args, dist):
    """The reference arm for decode attention: the oracle, one (token, layer)
    per step over the same 30-layer mix, on one host core."""
    if dist.rank != 0:
        return 0
    import oracle
    from expert_streaming_decode_b200 import synth
    O = oracle.get()
    A = synth.GEMMA4_ATTN
    layers = _attn_layers(A)
    nl = len(layers)
    kv = [synth.attn_kv(args.seed, l, A.Hkv, cap, A.hd) for l, (cap, _) in enumerate(layers)]
    scale = 1.0 / math.sqrt(A.hd)

    def step(i):
        t, l = divmod(i, nl)
        cap, n = layers[l]
        O.attn_decode(synth.attn_query(args.seed, t, l, A.Hq, A.hd), kv[l][0], kv[l][1], cap, n, scale)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.warmup, args.warmup + args.steps):
        step(i)
    el = time.perf_counter() - t0
    v = args.steps / nl / el
    line = {"impl": "reference", "metric": METRIC_ATTN, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "attn_decode", "layers": nl, "heads_q": A.Hq, "heads_kv": A.Hkv,
                       "head_dim": A.hd, "window": A.window, "context": A.context,
                       "step": "one (token, layer) of the 30-layer mix"},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": f"{args.steps} (token, layer) steps after {args.warmup} warm-up steps"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_attn(args, dist):
    """Decode attention for every layer of one token per step, from resident
    KV caches (378 MB, larger than L2), replayed as a CUDA graph."""
    import torch
    from expert_streaming_decode_b200 import moe, synth
    A = synth.GEMMA4_ATTN
    layers = _attn_layers(A)
    nl = len(layers)
    scale = 1.0 / math.sqrt(A.hd)
    seed = args.seed + 23 * dist.rank
    t0 = time.perf_counter()
    K_, V_ = [], []
    for l, (cap, _) in enumerate(layers):
        k, v = synth.attn_kv(seed, l, A.Hkv, cap, A.hd)
        K_.append(torch.from_numpy(k.view(np.int16)).cuda())
        V_.append(torch.from_numpy(v.view(np.int16)).cuda())
    W, Ks = args.warmup, args.steps
    qs = np.stack([np.stack([synth.attn_query(seed, t, l, A.Hq, A.hd) for l in range(nl)]) for t in range(W + Ks)])
    gen_s = time.perf_counter() - t0
    qs_dev = torch.from_numpy(qs.view(np.int16)).cuda()
    q_buf = torch.empty_like(qs_dev[0])
    o = torch.empty((nl, A.Hq, A.hd), dtype=torch.float32, device="cuda")
    ws = torch.zeros(moe.attn_workspace_bytes(A.Hq, A.hd), dtype=torch.uint8, device="cuda")
    step_bytes = sum(_attn_bytes(A, cap, n) for cap, n in layers)

    def layers_pass(stream=None):
        for l, (cap, n) in enumerate(layers):
            moe.attn_decode(q_buf[l], K_[l], V_[l], A.Hq, A.Hkv, A.hd, cap, n, scale, o[l], ws, stream=stream)

    # one step = the step's queries into place + 30 launches, as a graph
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        layers_pass(side)  # first calls outside capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        layers_pass(side)
    torch.cuda.synchronize()

    def run(i0, n):
        for i in range(i0, i0 + n):
            q_buf.copy_(qs_dev[i], non_blocking=True)
            graph.replay()

    run(0, W)
    clocks = ClockSampler(dist.local)
    if not args.profile:
        clocks.start()
    torch.cuda.synchronize()
    dist.barrier()
    st = torch.cuda.current_stream()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(st)
    run(W, Ks)
    eb.record(st)
    torch.cuda.synchronize()
    dist.barrier()
    ms = dist.max(ea.elapsed_time(eb))
    clk = clocks.stop() if not args.profile else None

    # per-launch durations: event pairs around every launch on its stream
    kinds = {"sliding": [0.0, 0, 0], "full": [0.0, 0, 0]}
    kp = min(Ks, 32)
    evs = []
    for i in range(kp):
        q_buf.copy_(qs_dev[W + i])
        for l, (cap, n) in enumerate(layers):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            moe.attn_decode(q_buf[l], K_[l], V_[l], A.Hq, A.Hkv, A.hd, cap, n, scale, o[l], ws)
            b.record(st)
            evs.append(("full" if cap == A.context else "sliding", _attn_bytes(A, cap, n), a, b))
    torch.cuda.synchronize()
    for kind, byts, a, b in evs:
        kinds[kind][0] += a.elapsed_time(b)
        kinds[kind][1] += 1
        kinds[kind][2] += byts
    hbm_peak, peak_kind = peaks()
    kern = {k: {"ms_total": v[0], "launches": v[1], "bytes_per_launch": v[2] / max(1, v[1]),
                "us_per_launch": 1e3 * v[0] / max(1, v[1]), "gbs": v[2] / (v[0] * 1e-3) / 1e9}
            for k, v in kinds.items() if v[1]}
    # every kernel of the timed region is this one: its average duration there
    # is the step time over the step's launches (the step's query copy, a few
    # microseconds, is included, so this understates the kernel)
    ach = step_bytes / (ms / Ks * 1e-3) / 1e9

    tokens_all = dist.sum(Ks)
    line = {"metric": METRIC_ATTN, "value": tokens_all / (ms * 1e-3), "unit": "tokens/s", "n_gpus": dist.world,
            "steps": Ks, "warmup": W, "ms_per_step": ms / Ks, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "attn_decode", "layers": nl, "heads_q": A.Hq, "heads_kv": A.Hkv,
                       "head_dim": A.hd, "window": A.window, "context": A.context,
                       "layer_mix": "5 sliding-window (ring of 1024) then 1 full (linear 4096), x5",
                       "parallelism": f"replicas x{dist.world}",
                       "l2": f"working set > L2: {step_bytes / 1e6:.0f} MB of KV cache read per step",
                       "input_generation_s": gen_s},
            "roofline": {"bound": "hbm", "kernel": "attn_decode_kernel (all 30 launches of a step)",
                         "achieved": ach, "peak": hbm_peak, "unit": "GB/s", "frac": ach / hbm_peak,
                         "traffic": recorded_traffic("attn_decode", "traffic_attn.json", "bytes_per_step"),
                         "traffic_unit": "DRAM bytes per step (ncu)",
                         "peak_source": f"{peak_kind} hbm_gbs", "bytes_per_step": step_bytes,
                         "note": "achieved = algorithmic bytes per step / device time per step in the timed region"},
            "kernels": kern,
            "kernels_note": f"per-launch times from a separate pass of {kp} steps with an event pair around every "
                            "launch (serialised: no overlap between launches)",
            "gpu_launches": int(dist.sum(nl * Ks))}
    if clk:
        line["clocks"] = clk
    if not args.no_e2e:
        # through the API from host memory: the step's queries H2D, outputs D2H
        q_host = torch.from_numpy(qs.view(np.int16)).pin_memory()
        o_host = torch.empty((nl, A.Hq, A.hd), dtype=torch.float32).pin_memory()
        torch.cuda.synchronize()
        dist.barrier()
        ea.record(st)
        for i in range(W, W + Ks):
            q_buf.copy_(q_host[i], non_blocking=True)
            graph.replay()
            o_host.copy_(o, non_blocking=True)
        eb.record(st)
        torch.cuda.synchronize()
        dist.barrier()
        ms2 = dist.max(ea.elapsed_time(eb))
        line["e2e"] = {"value": tokens_all / (ms2 * 1e-3), "unit": "tokens/s",
                       "h2d_bytes_per_step": int(q_buf.numel() * 2), "d2h_bytes_per_step": int(o.numel() * 4),
                       "api": "moe_attn_decode x 30 per step (graph), queries copied from pinned host, outputs back"}
    if dist.rank == 0 and not args.no_cpu:
        line["cpu_baseline"] = attn_cpu_baseline(A, seed)
    del graph
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ main
def main():
    args = parse_args()
    from expert_streaming_decode_b200 import synth
    dims = synth.Dims(L=args.layers, S=args.slots)
    dist = Dist()
    if args.impl == "reference":
        dist.init("gloo")
        rc = run_reference_attn(args, dist) if args.workload == "attn_decode" else run_reference(args, dims, dist)
        dist.close()
        return rc

    import torch
    torch.cuda.set_device(dist.local)
    dist.init("nccl")
    if args.workload == "sweep":
        rc = run_sweep(args, dims, dist)
        dist.close()
        return rc
    if args.workload == "attn_decode":
        rc = run_attn(args, dist)
        dist.close()
        return rc
    T = args.batch if args.workload == "decode_resident" else (128 if args.workload == "prefill" else 1)
    if args.workload == "prefill" and args.steps == 240 and args.warmup == 16:
        args.steps, args.warmup = 4, 1  # a chunk is ~9 GB of cold fills: keep the default run short
    streaming = args.workload in ("decode_stream", "prefill")
    model = Model(args, dims, max_tokens=T, streaming=streaming, dist=dist)
    W, K = args.warmup, args.steps
    ntok = W + K
    xs = np.stack([synth.hidden_batch(args.seed + 17, range(i * T, i * T + T), 0, dims.D) for i in range(ntok)])
    x_dev = torch.from_numpy(xs.view(np.int16)).cuda()

    # ---- timed pass: inputs resident in HBM, no instrumentation; the cache
    # counters are read on the device (no host round trip per layer)
    runner = Runner(model, T, graph=not streaming)
    runner.cold_each_step = args.workload == "prefill"
    model.reset()
    runner.run(x_dev, W, 0)
    clocks = ClockSampler(dist.local)
    if not args.profile:
        clocks.start()
    st0 = model.ctx.stats() if streaming else None
    pf0 = moe_prefetch_stats(model)
    ms, launches = timed(dist, model, lambda: runner.run(x_dev, K, W))
    clk = clocks.stop() if not args.profile else None
    pf1 = moe_prefetch_stats(model)
    st1 = model.ctx.stats() if streaming else None

    # ---- kernel timing pass: event pairs around every kernel (this serialises
    # the kernels, so it is kept out of the pass above)
    kp = min(K, 32)
    model.reset()
    runner_p = Runner(model, T, graph=False)
    runner_p.cold_each_step = args.workload == "prefill"
    runner_p.run(x_dev, min(W, 2), 0)
    model.ctx.profile(True)
    ms_p, _ = timed(dist, model, lambda: runner_p.run(x_dev, kp, W))
    model.ctx.profile(False)
    prof = model.ctx.profile_read()

    tokens_all = dist.sum(K * T)
    value = tokens_all / (ms * 1e-3)
    layer_kernel = prof["layer"][1] > 0
    line = {"metric": METRIC_PREFILL if args.workload == "prefill" else METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": dist.world, "steps": K, "warmup": W,
            "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": ("fp16 tcgen05 MMA on dequantised int4 tiles, fp32 accumulation" if T >= 2 else
                      "int4 weights x 16-bit fixed-point activations (dp4a), fp32 accumulation"),
            "data": "synthetic"}
    cfg = {"workload": args.workload, "layers": args.layers, "batch": T, "slots": args.slots if streaming else None,
           "cache_policy": (args.policy + (f"_{args.decay_period}" if args.policy == "lfu_decay" else ""))
           if streaming else None,
           "miss_fill": (("layer kernel reads pinned host memory" if args.fill == "direct" and T == 1
                          else "copy engine") if streaming and not args.store_file else None),
           "prefetch_buffers": args.prefetch if streaming else None,
           "lookahead_layers": (args.lookahead if args.prefetch else None) if streaming else None,
           "store": (("file, O_DIRECT" if args.direct else "file, page cache") if args.store_file else "pinned host memory")
           if streaming else None,
           "zipf_s": args.zipf, "zipf_lambda": args.zipf_lambda if args.zipf > 0 else None,
           "tokens_per_rank": ntok * T, "parallelism": f"replicas x{dist.world}",
           "l2": ("working set > L2: 30 layers x (16 slots + shared) = 1.9 GB in HBM plus a 12.85 GB pinned store"
                  if streaming else "working set > L2: 12.85 GB of resident experts")}
    line["config"] = cfg

    # ---- kernel rooflines from the live kernel timings
    hbm_peak, peak_kind = peaks()
    n_layer_tok = kp * args.layers
    distinct = float(dims.K) if T == 1 else dims.E * (1 - (1 - dims.K / dims.E) ** T)
    gu_b, dn_b, router_b = model.token_bytes_hbm(distinct)
    kern = {}
    kinds = (("layer", gu_b + dn_b + router_b),) if layer_kernel else \
        (("gate_up", gu_b), ("down", dn_b), ("router", router_b))
    for kind, byts in kinds:
        tms, cnt = prof[kind]
        if cnt:
            kern[kind] = {"ms_total": tms, "launches": cnt, "bytes_per_layer_token": byts,
                          "us_per_launch": 1e3 * tms / cnt,
                          "gbs": byts * n_layer_tok / (tms * 1e-3) / 1e9}
    for kind in ("plan", "worklist", "harness"):
        tms, cnt = prof[kind]
        if cnt:
            kern[kind] = {"ms_total": tms, "launches": cnt}
    dom = "layer" if layer_kernel else max(("gate_up", "down"), key=lambda k: kern[k]["ms_total"])
    ach = kern[dom]["gbs"]
    gemm = T >= model.moe.lib.moe_gemm_min_tokens()
    kname = ("layer_decode_kernel (one launch per layer)" if layer_kernel else
             "grouped_gemm_kernel (tcgen05)" if gemm else "gemv_decode_kernel" if T == 1 else "stream_gemv_kernel")
    hbm_roof = {"bound": "hbm", "kernel": kname if layer_kernel else f"{kname} ({dom})",
                "achieved": ach, "peak": hbm_peak, "unit": "GB/s", "frac": ach / hbm_peak,
                "traffic": (recorded_traffic(f"{args.workload}:{dom}") if not gemm else None),
                "traffic_unit": "DRAM bytes per layer-token (ncu, profiles/traffic.json)",
                "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)" if peak_kind == "measured"
                else "fallback 6650 GB/s",
                "measured_in": f"a separate pass of {kp} steps with an event pair around every kernel launch"}
    if not streaming and T == 1:
        # the step-level rate of the timed pass (the graph keeps launches chained)
        step_bytes = args.layers * (gu_b + dn_b + router_b)
        hbm_roof["step_level"] = {"achieved": step_bytes / (ms / K * 1e-3) / 1e9,
                                  "frac": step_bytes / (ms / K * 1e-3) / 1e9 / hbm_peak,
                                  "bytes_per_step": step_bytes}
    line["roofline"] = hbm_roof
    if gemm:
        # the grouped GEMM's FLOPs: 2 * pairs * (3 * F * D) routed + 2 * T * (3 * FS * D) shared per layer
        flop_layer = 2.0 * T * dims.K * 3 * dims.F * dims.D + 2.0 * T * 3 * dims.FS * dims.D
        gemm_ms = kern["gate_up"]["ms_total"] + kern["down"]["ms_total"]
        # n_layer_tok counts layer-steps of T tokens each, and flop_layer already covers the T tokens
        tf = flop_layer * n_layer_tok / (gemm_ms * 1e-3) / 1e12
        pk = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["bf16_tflops"] if peak_kind == "measured" else 1590.0
        line["tensor"] = {"achieved_tflops": tf, "peak_tflops": pk, "frac": tf / pk,
                          "note": "fp16 tcgen05 MMAs (peak: bf16 dense, same rate as fp16); per-expert rows "
                                  f"average {T * dims.K / distinct:.1f} ({T} tokens over ~{distinct:.0f} experts), so "
                                  "the tensor pipe idles: the GEMM is bound by the weights' dequantisation and bytes"}
    line["kernels"] = kern
    line["kernels_note"] = (f"per-kernel times from a separate pass of {kp} steps with an event pair around every "
                            "kernel (serialised: no overlap between kernels)")
    if streaming:
        d_st = {k: st1[k] - st0[k] for k in st1}
        planned = max(1, d_st["planned"])
        miss_tok = d_st["miss_bytes"] / (K * T)
        pf_iss, pf_used = pf1[0] - pf0[0], pf1[1] - pf0[1]
        link_tok = miss_tok + (pf_iss - pf_used) / (K * T)  # bytes that crossed the host link per token
        peak_h2d = h2d_peak_gbs(torch)
        useful = miss_tok * (value / dist.world) / 1e9      # every missed expert crosses the link once
        line["hit_rate"] = 1.0 - d_st["misses"] / planned
        line["misses_per_token"] = d_st["misses"] / (K * T)
        line["miss_bytes_per_token"] = miss_tok
        if T == 1:
            # the identity miss bytes = (1 - hit) x layers x top-k x blob for one-token steps,
            # and the pages' repeat statistics of the routing (40 % / 57 %)
            want = (1.0 - line["hit_rate"]) * args.layers * dims.K * model.nb
            line["miss_bytes_check"] = {"measured": miss_tok, "from_hit_rate": want,
                                        "holds": abs(miss_tok - want) < 1.0}
            line["expert_repeat"] = {"next_token": d_st["repeat_prev"] / planned,
                                     "within_two_tokens": d_st["repeat_prev2"] / planned,
                                     "pages": {"next_token": 0.40, "within_two_tokens": 0.57},
                                     "note": "share of a token's selected experts (per layer) also selected by the "
                                             "previous token / one of the two previous tokens, over the timed tokens"}
        pcie = {"bound": "pcie", "achieved": useful, "peak": peak_h2d, "unit": "GB/s",
                "frac": useful / peak_h2d if peak_h2d else None, "traffic": link_tok,
                "traffic_unit": "bytes over the host link per token (misses not served from staged blobs + "
                                "look-ahead copies)",
                "peak_source": "measured in this run: 256 MiB pinned->device cudaMemcpyAsync, best of 6",
                "measured_in": "timed pass: missed-expert bytes per token (device counters) x tokens/s"}
        if args.workload == "decode_stream" and not args.store_file:
            # the miss path bounds the streamed decode: the link is the primary
            # roofline, the layer's HBM kernel the secondary
            line["roofline"] = {**pcie, "hbm_kernel": hbm_roof}
        else:
            line["pcie"] = pcie
        h2d_ms, h2d_n = prof["h2d"]
        if h2d_n:
            line["copy_batches"] = {"count": h2d_n, "ms_total": h2d_ms,
                                    "note": "batches of miss copies on the side stream, kernel timing pass"}
        if args.store_file:
            fstride = (model.nb + 4095) // 4096 * 4096
            paths = [os.path.join(args.store_file, f"layer{l:02d}.experts") for l in range(model.L)]
            fpk = file_read_peak_gbs(paths, fstride, args.direct)
            line["file_read"] = {"achieved": useful, "peak": fpk, "unit": "GB/s",
                                 "frac": useful / fpk if fpk else None,
                                 "peak_source": "measured in this run: 512 MiB of expert-sized positional reads, "
                                                "4 threads" + (", O_DIRECT" if args.direct else ", page cache"),
                                 "note": "misses are read from the expert files (positional reads into pinned "
                                         "staging, 4 in flight) and then copied"}
        if model.lookahead:
            line["prefetch"] = {"buffers": args.prefetch, "issued_bytes_per_token": pf_iss / (K * T),
                                "used_bytes_per_token": pf_used / (K * T),
                                "wasted_bytes_per_token": (pf_iss - pf_used) / (K * T),
                                "miss_bytes_served": pf_used / max(1, d_st["miss_bytes"]),
                                "note": "measured over the timed pass; staged blobs reach their slots device to "
                                        "device"}
    line["gpu_launches"] = int(dist.sum(launches))
    if clk:
        line["clocks"] = clk

    # ---- end to end through host buffers
    if not args.no_e2e and not args.profile:
        xh = torch.from_numpy(xs.view(np.int16)).pin_memory()
        yh = torch.empty((ntok, T, dims.D), dtype=torch.float32).pin_memory()
        model.reset()
        runner.run(None, W, 0, host_io=(xh, yh))
        ms2, _ = timed(dist, model, lambda: runner.run(None, K, W, host_io=(xh, yh)))
        line["e2e"] = {"value": dist.sum(K * T) / (ms2 * 1e-3), "unit": "tokens/s",
                       "h2d_bytes_per_step": T * dims.D * 2, "d2h_bytes_per_step": T * dims.D * 4,
                       "api": ("moe_layer_forward_next" if model.nexts is not None and T == 1 else "moe_layer_forward")
                              + f" x {args.layers} per step, input bf16 copied from pinned host, output fp32 copied back"}

    if dist.rank == 0 and dist.world == 1 and not args.no_cpu and not args.profile and args.workload == "decode_stream":
        line["cpu_baseline"] = cpu_baseline(args, dims)
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    model.ctx.close()
    model.close_files()
    dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
