#!/usr/bin/env python
"""Decode-step benchmark of Windowed-MTP draft + verify attention on B200.

One *step* is one speculative decode step of the attention hot path:
gamma draft forwards (each: append the draft token, then draft attention) +
L target layers of verify (each: write the gamma+1 new tokens, then causal
verify attention) + accept/rollback.  Two arms run on the same inputs and the
same seeded acceptance draws:

* windowed: draft attention over the compact sink + window ring (the method);
* native:   draft attention over the draft layer's full paged cache.

Default workload: batch 1, GQA 16 query / 2 KV heads, head_dim 256, page
size 64, context 1,048,576 tokens (about 2 GiB of bf16 KV per layer), S=4,
W=4096, gamma=3, L=10 verify layers of independent KV.  Inputs are seeded
synthetic tensors (synth module); all KV stays resident in HBM.

Each timed decode step of each arm replays as one CUDA graph (--eager: Python
launches), windowed and native steps alternating so both arms run under the
same clocks.

Prints ONE JSON line (rank 0).  `value` is the windowed arm's device time per
decode step in microseconds (max over ranks; lower is better).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "draft+verify attn us/decode step at 1M ctx; achieved HBM GB/s (native vs window)"
KV_BYTES_PER_TOKEN_HEAD = None  # set per workload: 2 (K,V) * D * 2 bytes


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["wmtp", "reference"], default="wmtp")
    ap.add_argument("--config", default="1m", choices=["tiny", "32k", "128k", "1m", "ragged4"])
    ap.add_argument("--gamma", type=int, default=3)
    ap.add_argument("--window", type=int, default=4096)
    ap.add_argument("--layers", type=int, default=None, help="verify layers (default: workload's)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--ctx", type=int, default=None, help="committed context length (default: the config's)")
    ap.add_argument("--sweep", action="store_true",
                    help="context x gamma x window sweep of native/windowed step time (one JSON line per point)")
    ap.add_argument("--eager", action="store_true",
                    help="time the steps as eager launches instead of one CUDA graph per decode step")
    ap.add_argument("--admission", action="store_true",
                    help="admit 1M-context requests into one fixed KV budget through the page allocator, "
                         "native vs windowed, then decode each arm's admitted batch (one JSON line)")
    ap.add_argument("--kv-budget-gb", type=float, default=130.0,
                    help="KV budget of --admission in GB (1e9 bytes)")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU; replicas, no data-path exchange)
# ---------------------------------------------------------------------------
def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_us_per_step(ms_max: float, steps: int, world: int) -> float:
    """Whole-job time per decode step: every rank runs `steps` steps of its own
    sequence; `ms_max` is the slowest rank's device time for them, so the job
    processed steps x world decode steps in ms_max."""
    return ms_max * 1000.0 / (steps * world)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock and throttle reasons sampled every few milliseconds during the
    timed region: NVML queries from a background thread (read-only), else
    `nvidia-smi -lms`."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    INTERVAL_S = 0.005

    def __init__(self, device_index, enabled: bool = True, uuid: str | None = None):
        self.proc = None
        self.thread = None
        self.idx = device_index
        self.lines = []
        self.samples = []
        self.max_mhz = None
        if not enabled:
            return
        try:
            import threading

            import pynvml
            pynvml.nvmlInit()
            h = None
            if uuid:
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
                except pynvml.NVMLError:
                    h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(int(device_index))
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self.nv = pynvml
            self.handle = h
            self.running = True
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        except Exception:  # no NVML: fall back to nvidia-smi
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={device_index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def _poll(self):
        nv, h = self.nv, self.handle
        while self.running:
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((float(sm), int(reasons)))
            except Exception:
                pass
            time.sleep(self.INTERVAL_S)

    def _stop_nvml(self):
        self.running = False
        self.thread.join(timeout=5)
        nv = self.nv
        # every clock-event reason NVML reports except idle (a leftover clock
        # lock shows as applications_clocks_setting)
        names = {"hw_slowdown": "HwSlowdown", "hw_thermal_slowdown": "HwThermalSlowdown",
                 "sw_thermal_slowdown": "SwThermalSlowdown", "sw_power_cap": "SwPowerCap",
                 "hw_power_brake_slowdown": "HwPowerBrakeSlowdown",
                 "applications_clocks_setting": "ApplicationsClocksSetting", "sync_boost": "SyncBoost",
                 "display_clock_setting": "DisplayClockSetting"}
        bits = {k: getattr(nv, "nvmlClocksEventReason" + v) for k, v in names.items()
                if hasattr(nv, "nvmlClocksEventReason" + v)}
        if not self.samples:
            return None
        reasons = sorted({name for _, r in self.samples for name, bit in bits.items() if r & bit})
        return {"sm_mhz": statistics.median(sm for sm, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml"}

    def stop(self):
        if self.thread is not None:
            return self._stop_nvml()
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1].split()[0]))
                mx = float(parts[2].split()[0])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi"}


# ---------------------------------------------------------------------------
# the workload
# ---------------------------------------------------------------------------
class Workload:
    """All device state of one replica: verify layers, the draft pool, the
    ring, and per-step inputs for warmup + timed steps.

    ``kv`` (optional) builds the paged caches instead of one seeded pool per
    layer: ``kv(workload, capacity_tokens) -> (verify caches, draft cache or
    None)``; without a draft cache the ring is filled with seeded tokens and
    only the windowed arm can run.  ``batch`` overrides the workload's batch
    (every sequence then has the same context)."""

    def __init__(self, args, rank, device, kv=None, batch=None):
        import numpy as np
        import torch

        import synth
        import speculative_decode_draft_b200 as w

        self.w = w
        self.torch = torch
        base = synth.workload(args.config)
        self.wl = base
        self.B = batch if batch is not None else base.batch
        self.Hq, self.Hkv, self.D, self.P = base.num_heads_q, base.num_heads_kv, base.head_dim, base.page_size
        self.G = self.Hq // self.Hkv
        self.S = base.sinks
        self.W = args.window if args.config in ("1m", "128k") else base.window
        self.gamma = args.gamma
        self.L = args.layers if args.layers is not None else base.verify_layers
        self.steps_total = args.steps + args.warmup
        # committed context per sequence at the first step (ragged4: one per sequence)
        self.n0s = [int(args.ctx)] * base.batch if args.ctx else [int(c) for c in base.context]
        if batch is not None:
            self.n0s = [max(self.n0s)] * batch
        self.n0 = max(self.n0s)
        seed = base.seed + 1000 * rank
        self.seed = seed
        dev = device
        self.dev = dev
        # acceptance draws (shared by both arms): a in 1..gamma+1
        self.accept = synth.accept_counts(seed, self.steps_total, self.B, self.gamma)
        # committed length at the start of each step
        self.n_at = np.zeros((self.steps_total + 1, self.B), dtype=np.int64)
        self.n_at[0] = self.n0s
        for s in range(self.steps_total):
            self.n_at[s + 1] = self.n_at[s] + self.accept[s]
        cap = int(self.n_at[-1].max()) + self.gamma + 2 + self.P
        self.p = w.params(self.Hq, self.Hkv, self.D, page_size=self.P, sinks=self.S, window=self.W,
                          gamma_max=self.gamma)
        kvs = base.kv_scale
        shuf = base.shuffle_pages
        self.draft = None
        if kv is None:
            # verify layers: independent random KV, n0 committed tokens each
            layers = [synth.paged_kv(seed + 10 + l, self.B, self.Hkv, self.D, self.P, self.n0s,
                                     cap, kvs, shuf, device=dev) for l in range(self.L)]
            # the draft layer's own KV (native arm reads it in full)
            self.draft = synth.paged_kv(seed + 5, self.B, self.Hkv, self.D, self.P, self.n0s, cap, kvs,
                                        shuf, device=dev)
            self.caches = [w.PagedCache(k.k_pool, k.v_pool, k.page_table, k.kv_len) for k in layers]
            self.draft_cache = w.PagedCache(self.draft.k_pool, self.draft.v_pool, self.draft.page_table,
                                            self.draft.kv_len)
            del layers
        else:
            self.caches, self.draft_cache = kv(self, cap)
        # per-step inputs
        T = self.steps_total
        g = torch.Generator(device=dev)
        g.manual_seed(seed + 99)

        def rnd(*shape):
            return torch.randn(shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
        self.q_draft = rnd(T, self.gamma, self.B, self.Hq, self.D)
        self.k_draft = rnd(T, self.gamma, self.B, 1, self.Hkv, self.D)
        self.v_draft = rnd(T, self.gamma, self.B, 1, self.Hkv, self.D)
        self.k_bonus = rnd(T, self.B, 1, self.Hkv, self.D)
        self.v_bonus = rnd(T, self.B, 1, self.Hkv, self.D)
        self.q_ver = rnd(T, self.L, self.B, self.gamma + 1, self.Hq, self.D)
        self.k_ver = rnd(T, self.L, self.B, self.gamma + 1, self.Hkv, self.D)
        self.v_ver = rnd(T, self.L, self.B, self.gamma + 1, self.Hkv, self.D)
        i32 = dict(dtype=torch.int32, device=dev)
        na = torch.from_numpy(self.n_at.astype(np.int32)).to(dev)
        ga = torch.arange(self.gamma, dtype=torch.int32, device=dev)
        self.len_draft = (na[:T, None, :] + ga[None, :, None] + 1).contiguous()      # [T, gamma, B]
        self.pos_draft = (na[:T, None, :] + ga[None, :, None]).contiguous()          # [T, gamma, B]
        self.len_ver = (na[:T] + self.gamma + 1).contiguous()                       # [T, B]
        self.pos_ver = na[:T].contiguous()                                          # [T, B]
        acc = torch.from_numpy(self.accept).to(dev)
        self.trunc_to = (na[:T] + torch.clamp(acc, max=self.gamma)).to(torch.int32).contiguous()
        self.n_bonus = (acc == self.gamma + 1).to(torch.int32).contiguous()
        self.one = torch.ones(self.B, **i32)
        self.status = w.new_status(dev)
        # outputs (fp32 output mode, allocated once)
        f32 = dict(dtype=torch.float32, device=dev)
        self.o_draft = torch.empty(self.B, self.Hq, self.D, **f32)
        self.l_draft = torch.empty(self.B, self.Hq, **f32)
        self.o_ver = torch.empty(self.B, self.gamma + 1, self.Hq, self.D, **f32)
        self.l_ver = torch.empty(self.B, self.gamma + 1, self.Hq, **f32)
        # ring of the windowed arm, filled from the draft layer's history (or
        # with seeded tokens when there is no paged draft layer)
        self.ring = w.Ring.allocate(self.p, self.B, dev)
        if self.draft is not None:
            kd = torch.zeros(self.B, self.n0, self.Hkv, self.D, dtype=torch.bfloat16, device=dev)
            vd = torch.zeros_like(kd)
            for b in range(self.B):
                k, v = synth.dense_from_paged(self.draft, b, self.n0s[b])
                kd[b, :self.n0s[b]].copy_(k)
                vd[b, :self.n0s[b]].copy_(v)
            w.ring_append(self.p, self.ring, kd, vd, torch.tensor(self.n0s, **i32), status=self.status)
            del kd, vd
        else:
            from speculative_decode_draft_b200.timing import fill_ring_to
            fill_ring_to(self.p, self.ring, self.n0, seed + 6, dev)
        torch.cuda.synchronize()
        ver_pages = self.caches[0].page_table.shape[1]
        draft_pages = self.draft_cache.page_table.shape[1] if self.draft_cache is not None else 1
        self.workspace = torch.empty(max(
            w.workspace_bytes("full", self.p, self.B, max_pages=draft_pages),
            w.workspace_bytes("verify", self.p, self.B, num_q=self.gamma + 1, max_pages=ver_pages),
            w.workspace_bytes("windowed", self.p, self.B),
            w.workspace_bytes("windowed_paged", self.p, self.B, max_pages=draft_pages)),
            dtype=torch.uint8, device=dev)

    # -- kernel launches of one step (for gpu_launches)
    def launches_per_step(self, arm: str) -> int:
        """Library kernels one decode step launches: per draft an append (ring
        or paged write), the attention and its combine; per verify layer the
        verify (which writes its new tokens itself on the tcgen05 path, else
        after a paged write) and its combine; the windowed arm's final ring
        append (accept / rollback)."""
        rows = (self.gamma + 1) * self.Hq // self.Hkv
        tc = self.D == 256 and self.gamma + 1 >= 2 and 9 <= rows <= 128
        n = self.gamma * 3 + self.L * (2 if tc else 3)
        return n + 1 if arm == "windowed" else n

    # -- one decode step; `ev` collects (kind, start_event, end_event)
    # names of the per-step input tensors (first dimension: the step)
    STEP_INPUTS = ("q_draft", "k_draft", "v_draft", "k_bonus", "v_bonus", "q_ver", "k_ver", "v_ver",
                   "len_draft", "pos_draft", "len_ver", "pos_ver", "trunc_to", "n_bonus")

    def step_inputs(self, s: int) -> dict:
        """This step's inputs: queries, new K/V, lengths and positions, the
        rollback targets and bonus-token counts drawn from the acceptance."""
        return {name: getattr(self, name)[s] for name in self.STEP_INPUTS}

    def step(self, s: int, arm: str, ev=None, inputs=None, external_events: bool = False, outputs=None):
        """One decode step.  ``inputs`` (a dict like ``step_inputs``) replaces
        the resident inputs of step ``s``; ``outputs`` (``{"draft": [gamma,
        ...], "verify": [L, ...]}`` device tensors) are written by the
        attention calls themselves in place of the resident output buffers.
        With ``ev`` one draft call and one
        verify call of the step (draft s mod gamma, layer s mod L) are
        bracketed by an event pair: an event node between two kernels ends the
        second one's programmatic overlap with the first, so the other calls
        keep theirs."""
        torch, w = self.torch, self.w

        def E(**kw):  # events inside a captured graph must be graph nodes
            return torch.cuda.Event(external=external_events, **kw)
        x = inputs if inputs is not None else self.step_inputs(s)
        ev_all = ev
        o_draft = (lambda j: outputs["draft"][j]) if outputs is not None else (lambda j: self.o_draft)
        o_ver = (lambda l: outputs["verify"][l]) if outputs is not None else (lambda l: self.o_ver)
        for j in range(self.gamma):
            ev = ev_all if j == s % self.gamma else None
            if arm == "windowed":
                w.ring_append(self.p, self.ring, x["k_draft"][j], x["v_draft"][j], self.one,
                              speculative=True, status=self.status)
                a = E(enable_timing=True) if ev is not None else None
                if a is not None:
                    a.record()
                w.draft_attn_windowed(self.p, x["q_draft"][j], self.ring, out=o_draft(j), lse=self.l_draft,
                                      workspace=self.workspace, status=self.status)
            else:
                self.draft_cache.kv_len = x["len_draft"][j]
                w.paged_write(self.p, self.draft_cache, x["pos_draft"][j], x["k_draft"][j], x["v_draft"][j],
                              status=self.status)
                a = E(enable_timing=True) if ev is not None else None
                if a is not None:
                    a.record()
                w.draft_attn_full(self.p, x["q_draft"][j], self.draft_cache, out=o_draft(j), lse=self.l_draft,
                                  workspace=self.workspace, status=self.status)
            if ev is not None:
                bnd = E(enable_timing=True)
                bnd.record()
                ev.append(("draft", a, bnd))
        for l in range(self.L):
            ev = ev_all if l == s % self.L else None
            c = self.caches[l]
            c.kv_len = x["len_ver"]
            a = E(enable_timing=True) if ev is not None else None
            if a is not None:
                a.record()
            # the layer's gamma+1 new tokens are written by the verify call
            # itself (positions len_ver - gamma - 1 = pos_ver ..)
            w.verify_attn_append(self.p, x["q_ver"][l], x["k_ver"][l], x["v_ver"][l], c, out=o_ver(l),
                                 lse=self.l_ver, workspace=self.workspace, status=self.status)
            if ev is not None:
                bnd = E(enable_timing=True)
                bnd.record()
                ev.append(("verify", a, bnd))
        if arm == "windowed":
            w.ring_append(self.p, self.ring, x["k_bonus"], x["v_bonus"], x["n_bonus"],
                          truncate_to=x["trunc_to"], status=self.status)

    def snapshot_ring(self):
        r = self.ring
        return [t.clone() for t in (r.k, r.v, r.tags, r.len, r.committed, r.undo_k, r.undo_v, r.undo_tags)]

    def restore_ring(self, snap):
        r = self.ring
        for dst, src in zip((r.k, r.v, r.tags, r.len, r.committed, r.undo_k, r.undo_v, r.undo_tags), snap):
            dst.copy_(src)


def algorithmic_bytes(wl, kind: str, ctxs) -> float:
    """Bytes a call must move with committed contexts `ctxs` (one per
    sequence): K and V of every attended token for every KV head, plus
    queries, page-table entries and fp32 outputs."""
    kvb = 2 * wl.Hkv * wl.D * 2
    qn = wl.gamma + 1 if kind == "verify" else 1
    q_bytes = len(ctxs) * qn * wl.Hq * wl.D * 2
    o_bytes = len(ctxs) * qn * wl.Hq * (wl.D + 1) * 4
    total = q_bytes + o_bytes
    for ctx in ctxs:
        if kind == "windowed":
            total += min(ctx, wl.S + wl.W) * (kvb + 4)
        else:
            total += ctx * kvb + math.ceil(ctx / wl.P) * 4
    return total


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline, not target)
# ---------------------------------------------------------------------------
ORACLE_CHUNK = 65536  # tokens per chunk of the oracle's full-context units


class OracleUnits:
    """The fp64 oracle timed on one unit of each kind at the workload's full
    context: one verify layer (gamma+1 causal queries), one native draft (one
    query over the whole cache) and one windowed draft (one query over S + W
    ring entries), every KV head, sequence 0 of the workload.

    The context is processed in 64K-token chunks: per chunk and KV head one
    ``oracle.attend_prefixes`` call (all query rows of the head, each with its
    causal limit inside the chunk), then ``oracle.splitkv_combine`` over the
    chunks -- both oracle functions, pinned by the oracle's tests.  Only the
    oracle calls are timed; drawing the seeded bf16 K/V and widening each
    chunk to fp64 are not.  A decode step is modelled from the measured units
    as gamma x draft + L x verify (windowed or native draft)."""

    def __init__(self, args):
        import torch

        import synth
        base = synth.workload(args.config)
        self.Hq, self.Hkv, self.D = base.num_heads_q, base.num_heads_kv, base.head_dim
        self.G = self.Hq // self.Hkv
        self.S = base.sinks
        self.W = args.window if args.config in ("1m", "128k") else base.window
        self.gamma = args.gamma
        self.L = args.layers if args.layers is not None else base.verify_layers
        self.ctxs = [int(args.ctx)] * base.batch if args.ctx else [int(c) for c in base.context]
        self.n = self.ctxs[0] + self.gamma + 1  # sequence 0, the verify block appended
        self.scale = 1.0 / math.sqrt(self.D)
        # seeded N(0, 1) values rounded to bf16 (numpy's generator: fast on the
        # host for the 1M context), K/V of one layer kept as bf16
        import numpy as np
        rng = np.random.default_rng(base.seed + 4242)

        def bf16(*shape):
            return torch.from_numpy(rng.standard_normal(shape, dtype=np.float32)).to(torch.bfloat16)
        self.k = bf16(self.n, self.Hkv, self.D)
        self.v = bf16(self.n, self.Hkv, self.D)
        self.qv = bf16(self.gamma + 1, self.Hq, self.D).double().numpy()
        self.qd = bf16(self.Hq, self.D).double().numpy()
        self._f64 = {}

    def _chunk(self, c0, c1, kvh):
        # widened once, then reused by every unit and step (8.6 GB of fp64 at 1M)
        key = (c0, kvh)
        if key not in self._f64:
            self._f64[key] = (self.k[c0:c1, kvh].double().numpy(), self.v[c0:c1, kvh].double().numpy())
        return self._f64[key]

    def _full_context(self, qs_of, limits):
        """attend_prefixes per chunk + splitkv_combine; returns timed seconds."""
        import numpy as np

        import oracle
        t = 0.0
        for kvh in range(self.Hkv):
            qs = qs_of(kvh)
            parts_o, parts_l = [], []
            for c0 in range(0, self.n, ORACLE_CHUNK):
                c1 = min(self.n, c0 + ORACLE_CHUNK)
                K, V = self._chunk(c0, c1, kvh)
                lengths = np.clip(np.asarray(limits) - c0, 0, c1 - c0)
                t0 = time.perf_counter()
                o, lse = oracle.attend_prefixes(qs, K, V, lengths, self.scale)
                t += time.perf_counter() - t0
                parts_o.append(o)
                parts_l.append(lse)
            t0 = time.perf_counter()
            oracle.splitkv_combine(np.stack(parts_o, axis=1), np.stack(parts_l, axis=1))
            t += time.perf_counter() - t0
        return t

    def verify_s(self):
        G, Qn = self.G, self.gamma + 1
        limits = [self.n - Qn + i + 1 for i in range(Qn) for _ in range(G)]  # row i * G + g: query i
        return self._full_context(lambda kvh: self.qv[:, kvh * G:(kvh + 1) * G].reshape(Qn * G, self.D), limits)

    def draft_native_s(self):
        G = self.G
        return self._full_context(lambda kvh: self.qd[kvh * G:(kvh + 1) * G], [self.n] * G)

    def draft_windowed_s(self):
        import numpy as np

        import oracle
        G = self.G
        pos = oracle.window_positions(self.n, self.S, self.W)
        t = 0.0
        for kvh in range(self.Hkv):
            K = self.k[pos, kvh].double().numpy()
            V = self.v[pos, kvh].double().numpy()
            t0 = time.perf_counter()
            oracle.attend_prefixes(self.qd[kvh * G:(kvh + 1) * G], K, V, np.full(G, len(pos)), self.scale)
            t += time.perf_counter() - t0
        return t

    def step_model(self):
        """Measured unit times and the modelled decode step (us) of both arms;
        every sequence of the workload costs its own context's share."""
        tv, tn, tw = self.verify_s(), self.draft_native_s(), self.draft_windowed_s()
        f = sum(self.ctxs) / self.ctxs[0]  # other sequences: same per-token cost at their own length
        return {"verify_s": tv, "draft_native_s": tn, "draft_windowed_s": tw,
                "native_us": (self.gamma * tn + self.L * tv) * f * 1e6,
                "windowed_us": (self.gamma * tw * len(self.ctxs) + self.L * tv * f) * 1e6,
                "work_s": tv + tn + tw}

    def sample_desc(self):
        return (f"fp64 numpy oracle, one verify layer ({self.gamma + 1} causal queries), one native draft and one "
                f"windowed draft (S={self.S}, W={self.W}) at the full context of {self.n} tokens, every KV head "
                f"({self.Hq}q/{self.Hkv}kv, D={self.D}), in {ORACLE_CHUNK}-token chunks (attend_prefixes per chunk, "
                f"splitkv_combine); step modelled as gamma x draft + {self.L} x verify"
                + ("" if len(self.ctxs) == 1 else f", scaled to the {len(self.ctxs)} sequences' contexts"))


def cores_used():
    try:
        from threadpoolctl import threadpool_info
        th = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if th:
            return int(max(th))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


# DRAM traffic of one verify_tc_kernel launch from one ncu capture (--set
# full, 1 launch) of the 128K workload (batch 1, 16q/2kv heads, D=256, page
# 64, 131,072 + 4 tokens; about 3 GB on the device): dram__bytes_read.sum and
# dram__bytes_write.sum, and the K/V tokens that launch read.  Reads grow in
# proportion to the tokens read (every K/V byte crosses HBM once); the writes
# are the split partials, the same size at any context with the same split
# count (74 per KV head for batch 1).  So a launch reading `tokens` tokens is
# credited read_bytes * tokens / captured_tokens + write_bytes.  The figure is
# reported only while the kernel's code (its sources with comments and
# whitespace removed) hashes to the value it was captured on; otherwise
# roofline.traffic is null.
VERIFY_TRAFFIC = {
    "sources": ("speculative_decode_draft_b200/csrc/verify_tc.cuh", "speculative_decode_draft_b200/csrc/ptx.cuh"),
    "sha256": "0aa88727134350119405ddb7b47311b7bcd6131ac7c235e4beeac024cf25ef9f",
    "captured_on": "128k: verify_tc_kernel<3, 3, 64> with the fused append and P_lo in the spare lanes, "
                   "148 CTAs x 384 threads",
    "tokens": 131076,
    "read_bytes": 268724224,
    "write_bytes": 5498112,
}


def kernel_code_hash(root=None) -> str:
    """sha256 of the verify kernel's sources with comments and whitespace removed."""
    import hashlib
    import re
    h = hashlib.sha256()
    for rel in VERIFY_TRAFFIC["sources"]:
        with open(os.path.join(root or ROOT, rel)) as f:
            code = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
        code = re.sub(r"//[^\n]*", "", code)
        h.update(" ".join(code.split()).encode())
    return h.hexdigest()


def verify_traffic(tokens: int):
    """Captured DRAM bytes of one verify launch, scaled to a launch reading
    `tokens` K/V tokens; None if nothing was captured for this kernel code."""
    t = VERIFY_TRAFFIC
    if t["read_bytes"] is None or not t["tokens"] or kernel_code_hash() != t["sha256"]:
        return None
    return t["read_bytes"] * tokens / t["tokens"] + t["write_bytes"]


def staging_layout(shapes: dict, align: int = 256):
    """Byte offsets of named tensors packed into one flat staging buffer, each
    slot starting on an ``align``-byte boundary (the calls take 16-byte
    aligned pointers); ``shapes`` maps a name to ``(numel, element_size)``.
    Returns ``(offsets, total_bytes)``."""
    offs, off = {}, 0
    for name, (numel, esize) in shapes.items():
        offs[name] = off
        off += -(-numel * esize // align) * align
    return offs, off


def workload_desc(args) -> str:
    """The workload string of `config`, shared by both arms."""
    import synth
    base = synth.workload(args.config)
    W = args.window if args.config in ("1m", "128k") else base.window
    L = args.layers if args.layers is not None else base.verify_layers
    ctx = args.ctx if args.ctx else "/".join(str(c) for c in base.context)
    return (f"{args.config}: batch {base.batch}, {base.num_heads_q}q/{base.num_heads_kv}kv heads, "
            f"D={base.head_dim}, page {base.page_size}, ctx {ctx}, S={base.sinks}, W={W}, "
            f"gamma={args.gamma}, {L} verify layers")


def run_reference(args):
    """The reference arm: the fp64 CPU oracle on the host cores, per decode
    step of the same workload (each step measures one verify layer, one native
    draft and one windowed draft at the full context, and models the step from
    them); rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    units = OracleUnits(args)
    per = []
    for i in range(args.warmup + args.steps):
        r = units.step_model()
        if i >= args.warmup:
            per.append(r)
    v = statistics.median(x["windowed_us"] for x in per)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "us/step", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": v / 1000.0, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(args),
                   "native_us_per_step": statistics.median(x["native_us"] for x in per),
                   "verify_s_per_layer": statistics.median(x["verify_s"] for x in per),
                   "draft_native_s": statistics.median(x["draft_native_s"] for x in per),
                   "draft_windowed_s": statistics.median(x["draft_windowed_s"] for x in per)},
        "cpu_baseline": {"value": v, "unit": "us/step", "cores": cores_used(), "kind": "oracle",
                         "sample": units.sample_desc()},
        "e2e": {"value": v, "unit": "us/step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def time_arms(args, wk, world: int, make_clocks=None) -> dict:
    """Warm up both arms, capture each timed step as a CUDA graph (unless
    --eager), then time K steps of each arm, windowed and native alternating,
    between a barrier + synchronize on both sides.  Returns per-arm device ms
    (max over ranks), per-call means by kind (us) and the clock record."""
    import torch
    # ---------------- warmup (both arms)
    for s in range(args.warmup):
        wk.step(s, "native")
        wk.step(s, "windowed")
    torch.cuda.synchronize()
    ring_after_warmup = wk.snapshot_ring()
    if int(wk.status.item()) != 0:
        raise SystemExit(f"device status {int(wk.status.item()):#x} during warmup")

    # One CUDA graph per timed decode step and arm (the step's ~40 library
    # launches replay without host gaps); --eager launches them from Python.
    # Each step brackets one draft call and one verify call with events (the
    # per-call means); the other calls run as the product runs them.
    graphs = {}
    if not args.eager:
        for arm in ("windowed", "native"):
            graphs[arm] = []
            for s in range(args.warmup, args.warmup + args.steps):
                evs = []
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    wk.step(s, arm, ev=evs, external_events=True)
                graphs[arm].append((g, evs))
        torch.cuda.synchronize()

    def timed_interleaved():
        """K decode steps of each arm, alternating windowed and native step by
        step so both arms see the same clocks and power state; each step is
        bracketed by its own events and an arm's time is the sum of its steps."""
        evs = {"windowed": [], "native": []}
        spans = {"windowed": [], "native": []}
        wk.restore_ring(ring_after_warmup)
        barrier(world)
        torch.cuda.synchronize()
        for i, s in enumerate(range(args.warmup, args.warmup + args.steps)):
            for arm in ("windowed", "native"):
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record()
                if graphs:
                    g, gev = graphs[arm][i]
                    g.replay()
                    evs[arm].extend(gev)
                else:
                    wk.step(s, arm, ev=evs[arm])
                b.record()
                spans[arm].append((a, b))
        torch.cuda.synchronize()
        barrier(world)
        ms = {arm: sum(a.elapsed_time(b) for a, b in spans[arm]) for arm in spans}
        return ms, evs

    # the windowed arm advances the ring; the native arm must not see a
    # different ring, and neither reads the other's state
    clocks = make_clocks() if make_clocks else None
    ms_arm, ev_arm = timed_interleaved()
    clk = clocks.stop() if clocks else None
    ms_win = max_over_ranks(ms_arm["windowed"], world)
    ms_nat = max_over_ranks(ms_arm["native"], world)
    ev_win, ev_nat = ev_arm["windowed"], ev_arm["native"]

    def per_kind(evs):
        out = {}
        for kind, a, b in evs:
            out.setdefault(kind, []).append(a.elapsed_time(b) * 1000.0)
        return {k: statistics.mean(v) for k, v in out.items()}

    return {"ms_win": ms_win, "ms_nat": ms_nat, "k_win": per_kind(ev_win), "k_nat": per_kind(ev_nat),
            "clocks": clk, "ring_after_warmup": ring_after_warmup}


def run_sweep(args, rank: int, world: int, dev) -> int:
    """The pages' windowing wedge, step^native / step^windowed - 1, over
    context, draft depth and window (one JSON line per point, rank 0)."""
    import copy

    import torch
    contexts = (2048, 8192, 32768, 131072, 524288, 1048576)
    points = [(c, g, 2048) for c in contexts for g in (1, 3, 5, 8)]
    points += [(c, 3, W) for c in (32768, 1048576) for W in (1024, 4096, 8192)]
    for ctx, gamma, window in points:
        a = copy.copy(args)
        a.config, a.ctx, a.gamma, a.window = "1m", ctx, gamma, window
        wk = Workload(a, rank, dev)
        r = time_arms(a, wk, world)
        if int(wk.status.item()) != 0:
            raise SystemExit(f"device status {int(wk.status.item()):#x} at ctx {ctx} gamma {gamma} W {window}")
        win = whole_job_us_per_step(r["ms_win"], a.steps, world)
        nat = whole_job_us_per_step(r["ms_nat"], a.steps, world)
        if rank == 0:
            print(json.dumps({"sweep": True, "ctx": ctx, "gamma": gamma, "window": window, "layers": wk.L,
                              "windowed_us": win, "native_us": nat, "wedge": nat / win - 1.0,
                              "bytes_implied_wedge": gamma * (1.0 - min(ctx, 4 + window) / ctx) / wk.L,
                              "draft_windowed_us": r["k_win"]["draft"], "draft_native_us": r["k_nat"]["draft"],
                              "verify_us": r["k_win"]["verify"]}), flush=True)
        del wk, r
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return 0


def time_single_arm(args, wk, arm: str, world: int) -> dict:
    """Warm up one arm, capture each timed step as a CUDA graph, time K steps
    between a barrier + synchronize on both sides (max over ranks)."""
    import torch
    for s in range(args.warmup):
        wk.step(s, arm)
    torch.cuda.synchronize()
    graphs = []
    for s in range(args.warmup, args.warmup + args.steps):
        evs = []
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            wk.step(s, arm, ev=evs, external_events=True)
        graphs.append((g, evs))
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for g, _ in graphs:
        g.replay()
    b.record()
    torch.cuda.synchronize()
    barrier(world)
    per = {}
    for _, evs in graphs:
        for kind, e0, e1 in evs:
            per.setdefault(kind, []).append(e0.elapsed_time(e1) * 1000.0)
    ms = max_over_ranks(a.elapsed_time(b), world)
    del graphs
    return {"us_per_step": ms * 1000.0 / args.steps, "per_call_us": {k: statistics.mean(v) for k, v in per.items()}}


def run_admission(args, rank: int, world: int, dev) -> int:
    """The capacity side of Windowed-MTP (arxivlens view, Abstract: the ring
    frees the draft layer's otherwise dead KV pool, room for one more
    concurrent 1M request).  One fixed KV budget becomes one pool of pages;
    requests of the 1M workload are admitted through the page allocator
    (wmtp_pool_alloc, all of a request's pages at once) until it refuses:
    a native request takes every paged layer's pages (10 target + 1 draft), a
    windowed one the target layers' pages plus pages worth its ring (the ring
    itself is a separate tensor of that size).  Each arm's admitted batch is
    then decoded with page tables taken from the allocator."""
    import torch

    import synth
    import speculative_decode_draft_b200 as w
    base = synth.workload("1m")
    ctx = int(args.ctx) if args.ctx else base.context[0]
    Hq, Hkv, D, P, S = base.num_heads_q, base.num_heads_kv, base.head_dim, base.page_size, base.sinks
    L = args.layers if args.layers is not None else base.verify_layers
    gamma, W = args.gamma, args.window
    budget = int(args.kv_budget_gb * 1e9)
    page_bytes = 2 * Hkv * P * D * 2                      # K and V of one page, bf16
    num_pages = budget // page_bytes
    growth = (args.steps + args.warmup) * (gamma + 1)     # tokens the timed and warm-up steps can add
    p = w.params(Hq, Hkv, D, page_size=P, sinks=S, window=W, gamma_max=gamma)
    plan = {arm: w.plan_admission(p, ctx + growth, L, 1, arm == "windowed", budget)
            for arm in ("native", "windowed")}
    pages_layer = plan["native"]["pages_per_layer"]
    ring_bytes = plan["windowed"]["draft_bytes"]
    ring_pages = -(-ring_bytes // page_bytes)
    # the pool: every page filled with seeded bf16 values once
    k_pool = torch.empty(num_pages, Hkv, P, D, dtype=torch.bfloat16, device=dev)
    v_pool = torch.empty_like(k_pool)
    g = torch.Generator(device=dev)
    g.manual_seed(base.seed + 1000 * rank + 77)
    step = max(1, (1 << 30) // (Hkv * P * D * 2))
    for t in (k_pool, v_pool):
        for i in range(0, num_pages, step):
            t[i:i + step].normal_(generator=g)
    pool = w.PagePool(num_pages)
    result = {"kv_budget_bytes": budget, "pool_pages": num_pages, "page_bytes": page_bytes,
              "context": ctx, "target_layers": L, "draft_layers": 1, "gamma": gamma, "window": W,
              "pages_per_layer": pages_layer, "ring_pages": ring_pages}
    for arm in ("native", "windowed"):
        need = (L + 1) * pages_layer if arm == "native" else L * pages_layer + ring_pages
        admitted = []
        while True:
            try:
                admitted.append(pool.alloc(need))
            except w.WmtpError:
                break
        B = len(admitted)
        result[f"{arm}_requests"] = B
        result[f"{arm}_planned_requests"] = plan[arm]["max_requests"]
        result[f"{arm}_pages_used"] = B * need
        if B == 0:
            continue

        def kv(wk, cap, admitted=admitted, arm=arm):
            # every position a step reads or writes lies in the request's pages
            assert -(-(int(wk.n_at[-1].max()) + gamma + 1) // P) <= pages_layer
            lens = torch.tensor(wk.n0s, dtype=torch.int32, device=dev)

            def table(l):
                rows = [req[l * pages_layer:(l + 1) * pages_layer] for req in admitted]
                return torch.tensor(rows, dtype=torch.int32, device=dev)
            caches = [w.PagedCache(k_pool, v_pool, table(l), lens.clone()) for l in range(L)]
            draft = w.PagedCache(k_pool, v_pool, table(L), lens.clone()) if arm == "native" else None
            return caches, draft
        a = argparse.Namespace(**vars(args))
        a.config, a.ctx = "1m", ctx
        wk = Workload(a, rank, dev, kv=kv, batch=B)
        r = time_single_arm(a, wk, arm, world)
        torch.cuda.synchronize()
        result[f"{arm}_step_us"] = r["us_per_step"]
        result[f"{arm}_verify_us_per_layer"] = r["per_call_us"].get("verify")
        result[f"{arm}_draft_us"] = r["per_call_us"].get("draft")
        acc = wk.accept[args.warmup:].sum() / args.steps  # accepted tokens per step, whole batch
        result[f"{arm}_accepted_tokens_per_step"] = float(acc)
        result[f"{arm}_tokens_per_s"] = float(acc) / (r["us_per_step"] * 1e-6)
        result[f"{arm}_device_status"] = int(wk.status.item())
        del wk
        for req in admitted:
            pool.release(req)
        torch.cuda.empty_cache()
    if rank == 0:
        line = {"admission": True, "metric": METRIC, "unit": "us/step", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "dtype": "bf16", "data": "synthetic", **result}
        if result.get("native_tokens_per_s") and result.get("windowed_tokens_per_s"):
            line["windowed_over_native_throughput"] = result["windowed_tokens_per_s"] / result["native_tokens_per_s"]
        print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    import torch

    import speculative_decode_draft_b200 as w
    from speculative_decode_draft_b200 import build
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    rank, world, local = dist_setup(args)
    build.build()
    w.load()
    dev = torch.device("cuda", torch.cuda.current_device())
    if args.sweep:
        return run_sweep(args, rank, world, dev)
    if args.admission:
        return run_admission(args, rank, world, dev)
    free_bytes, _ = torch.cuda.mem_get_info()  # before the workload's own buffers
    wk = Workload(args, rank, dev)
    stream = torch.cuda.current_stream()

    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except (AttributeError, RuntimeError):
        uuid = None
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    smi_id = vis.split(",")[torch.cuda.current_device()].strip() if vis else str(torch.cuda.current_device())
    r = time_arms(args, wk, world,
                  lambda: ClockSampler(smi_id, enabled=not args.no_clocks and rank == 0, uuid=uuid))
    ms_win, ms_nat, k_win, k_nat, clk = r["ms_win"], r["ms_nat"], r["k_win"], r["k_nat"], r["clocks"]
    ring_after_warmup = r["ring_after_warmup"]
    ctx = wk.n0
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except (OSError, ValueError):
        pass
    hbm_peak = float(peaks.get("hbm_gbs", 6650.0))
    peak_src = "measured" if "hbm_gbs" in peaks else "fallback"

    class WL:  # shapes for the byte model
        B, Hq, Hkv, D, P, S, W, gamma = wk.B, wk.Hq, wk.Hkv, wk.D, wk.P, wk.S, wk.W, wk.gamma
    ver_bytes = algorithmic_bytes(WL, "verify", wk.n0s)
    nat_bytes = algorithmic_bytes(WL, "full", wk.n0s)
    win_bytes = algorithmic_bytes(WL, "windowed", wk.n0s)
    ver_gbs = ver_bytes / (k_win["verify"] * 1e-6) / 1e9
    nat_gbs = nat_bytes / (k_nat["draft"] * 1e-6) / 1e9
    win_gbs = win_bytes / (k_win["draft"] * 1e-6) / 1e9
    us_win = ms_win * 1000.0 / args.steps  # per rank
    us_nat = ms_nat * 1000.0 / args.steps

    # ---------------- end to end: host buffers, copies inside the timed region
    # Every step's inputs (queries, new K/V, lengths, positions, rollback
    # targets, bonus counts) start in pinned host memory and go to the device
    # in one copy; the attention calls write every output of the step into a
    # device staging buffer, which goes back to pinned host memory in one copy.
    e2e = None
    if not args.no_e2e:
        steps = range(args.warmup, args.warmup + args.steps)
        proto = wk.step_inputs(args.warmup)
        offs, off = staging_layout({k: (v.numel(), v.element_size()) for k, v in proto.items()})
        dev_flat = torch.empty(off, dtype=torch.uint8, device=dev)

        def views(flat):
            return {k: flat[offs[k]:offs[k] + v.numel() * v.element_size()].view(v.dtype).view(v.shape)
                    for k, v in proto.items()}
        host_in = {}
        for st_ in steps:
            flat = torch.empty(off, dtype=torch.uint8, pin_memory=True)
            for k, v in views(flat).items():
                v.copy_(wk.step_inputs(st_)[k])
            host_in[st_] = flat
        dev_in = views(dev_flat)
        n_d = wk.o_draft.numel()
        n_v = wk.o_ver.numel()
        out_flat = torch.empty(wk.gamma * n_d + wk.L * n_v, dtype=torch.float32, device=dev)
        outs = {"draft": out_flat[:wk.gamma * n_d].view((wk.gamma,) + tuple(wk.o_draft.shape)),
                "verify": out_flat[wk.gamma * n_d:].view((wk.L,) + tuple(wk.o_ver.shape))}
        host_out = {st_: torch.empty_like(out_flat, device="cpu", pin_memory=True) for st_ in steps}
        h2d = off
        d2h = out_flat.numel() * out_flat.element_size()
        wk.restore_ring(ring_after_warmup)
        barrier(world)
        torch.cuda.synchronize()
        st = torch.cuda.Event(enable_timing=True)
        en = torch.cuda.Event(enable_timing=True)
        st.record()
        for s in steps:
            dev_flat.copy_(host_in[s], non_blocking=True)
            wk.step(s, "windowed", inputs=dev_in, outputs=outs)
            host_out[s].copy_(out_flat, non_blocking=True)
        en.record()
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(st.elapsed_time(en), world)
        e2e = {"value": whole_job_us_per_step(ms_e2e, args.steps, world), "unit": "us/step",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "arm": "windowed",
               "path": "public Python API (eager launches); each step's inputs copied in from pinned host memory "
                       "in one transfer and its attention outputs copied back to pinned host memory in one"}
        del host_in, dev_in, outs, host_out, dev_flat, out_flat

    torch.cuda.synchronize()
    status = int(wk.status.item())

    # the windowed draft read through the page table (no ring) over the draft
    # layer's cache: ten calls captured in one CUDA graph, mean per call
    win_paged_us = None
    if not args.sweep:
        wk.draft_cache.kv_len = wk.len_draft[args.warmup, 0]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(10):
                w.draft_attn_windowed_paged(wk.p, wk.q_draft[args.warmup][0], wk.draft_cache, out=wk.o_draft,
                                            lse=wk.l_draft, workspace=wk.workspace, status=wk.status)
        g.replay()
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record()
        g.replay()
        b1.record()
        torch.cuda.synchronize()
        win_paged_us = b0.elapsed_time(b1) * 1000.0 / 10
        del g

    # verify (layer 0) and the native draft, ten calls back to back in one
    # CUDA graph: each call's launch and ramp overlap the previous call's tail
    # (programmatic launches), which the bracketed per-call times above cannot
    # show; context for the roofline, which uses the bracketed verify time
    b2b = None
    if not args.sweep:
        from speculative_decode_draft_b200.timing import graph_call_us
        s0 = args.warmup
        c0 = wk.caches[0]
        c0.kv_len = wk.len_ver[s0]
        ver_b2b = graph_call_us(lambda: w.verify_attn(wk.p, wk.q_ver[s0][0], c0, out=wk.o_ver, lse=wk.l_ver,
                                                      workspace=wk.workspace, status=wk.status))
        wk.draft_cache.kv_len = wk.len_draft[s0, 0]
        nat_b2b = graph_call_us(lambda: w.draft_attn_full(wk.p, wk.q_draft[s0][0], wk.draft_cache, out=wk.o_draft,
                                                          lse=wk.l_draft, workspace=wk.workspace,
                                                          status=wk.status))
        b2b = {"verify_us": ver_b2b, "verify_gbs": ver_bytes / (ver_b2b * 1e-6) / 1e9,
               "draft_native_us": nat_b2b, "draft_native_gbs": nat_bytes / (nat_b2b * 1e-6) / 1e9}

    # the windowed draft at 32K, 128K and 1M tokens of context (one sequence,
    # the ring in the state it has at that length): its time must not grow
    # with the context
    flat = None
    if not args.sweep:
        from speculative_decode_draft_b200.timing import fill_ring_to, graph_call_us
        flat = {}
        q1 = wk.q_draft[args.warmup][0][:1].contiguous()
        o1, l1 = wk.o_draft[:1], wk.l_draft[:1]
        rings = {}
        for c in (32768, 131072, 1048576):
            rings[c] = w.Ring.allocate(wk.p, 1, dev)
            fill_ring_to(wk.p, rings[c], c, seed=c, device=dev)
        # two interleaved rounds, the better time per context: the first
        # measurement after the timed region ran slower whichever context it was
        for _ in range(2):
            for c, ring in rings.items():
                t = graph_call_us(lambda: w.draft_attn_windowed(
                    wk.p, q1, ring, out=o1, lse=l1, workspace=wk.workspace, status=wk.status))
                flat[str(c)] = min(t, flat.get(str(c), math.inf))
        del rings
        torch.cuda.empty_cache()

    # a read-only streaming reference (torch's sum over 4 GiB; context for the
    # GB/s figures, not a peak the roofline divides by)
    read_gbs = None
    if not args.sweep:
        big = torch.ones(1 << 31, dtype=torch.bfloat16, device=dev)
        best = math.inf
        for _ in range(4):
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record()
            big.sum(dtype=torch.float32)
            a1.record()
            torch.cuda.synchronize()
            best = min(best, a0.elapsed_time(a1))
        read_gbs = big.numel() * 2 / (best * 1e-3) / 1e9
        del big
    status = int(wk.status.item())  # including the extra windowed-paged calls

    # the capacity side: requests of this context that the device's free
    # memory holds as KV, with the draft layer paged (native) or as a ring
    adm = {arm: w.plan_admission(wk.p, wk.n0, wk.L, 1, arm == "windowed", free_bytes)
           for arm in ("native", "windowed")}
    admission = {"kv_budget_bytes": free_bytes, "context": wk.n0, "target_layers": wk.L, "draft_layers": 1,
                 "native_requests": adm["native"]["max_requests"],
                 "windowed_requests": adm["windowed"]["max_requests"],
                 "reclaimed_fraction": 1 - adm["windowed"]["bytes_per_request"] / adm["native"]["bytes_per_request"]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        units = OracleUnits(args)
        r = units.step_model()
        cpu = {"value": r["windowed_us"], "unit": "us/step", "cores": cores_used(), "kind": "oracle",
               "sample": units.sample_desc() + f"; {r['work_s']:.1f} s of timed CPU work",
               "native_value": r["native_us"], "verify_s_per_layer": r["verify_s"],
               "draft_native_s": r["draft_native_s"], "draft_windowed_s": r["draft_windowed_s"]}
        del units

    if rank != 0:
        return 0
    value = whole_job_us_per_step(ms_win, args.steps, world)
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "us/step",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": us_win / 1000.0,
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": workload_desc(args),
            "l2": "inputs larger than L2 (verify reads ~2 GiB per layer per step); the ring stays L2-warm "
                  "between the draft steps of one decode step",
            "launch": "eager Python launches" if args.eager else "one CUDA graph per decode step and arm",
            "timing": "windowed and native steps alternate; each arm's time is the sum of its steps' CUDA-event "
                      "spans on the launching stream; per-call times from an event pair around one draft call "
                      "and one verify call of each timed step (draft s mod gamma, layer s mod L)",
            "native_us_per_step": us_nat,
            "windowed_us_per_step": us_win,
            "native_over_windowed": us_nat / us_win,
            "bytes_implied_ratio": (wk.gamma + wk.L) / wk.L,
            "draft_native_us": k_nat["draft"],
            "draft_windowed_us": k_win["draft"],
            "draft_windowed_paged_us": win_paged_us,
            "back_to_back": b2b,
            "draft_windowed_us_by_context": flat,
            "draft_windowed_spread_by_context": ((max(flat.values()) - min(flat.values())) / statistics.median(
                flat.values())) if flat else None,
            "verify_us_per_layer": k_win["verify"],
            "verify_us_per_layer_native_arm": k_nat["verify"],
            "draft_native_gbs": nat_gbs,
            "draft_windowed_gbs_l2": win_gbs,
            "verify_gbs": ver_gbs,
            "device_status": status,
            "read_stream_gbs_torch_sum": read_gbs,
            "admission": admission,
        },
        "roofline": {"bound": "hbm", "achieved": ver_gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": ver_gbs / hbm_peak,
                     "traffic": verify_traffic(sum(n + wk.gamma + 1 for n in wk.n0s)),
                     "kernel": "verify_tc_kernel: algorithmic bytes of one verify call / CUDA-event time of the "
                               "call (verify_tc_kernel + its split-KV combine)",
                     "algorithmic_bytes": ver_bytes, "peak_source": peak_src},
        "e2e": e2e,
        "gpu_launches": (wk.launches_per_step("windowed") + wk.launches_per_step("native")) * args.steps,
        "clocks": clk,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
