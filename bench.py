#!/usr/bin/env python
"""Benchmark: Q8_0 decode tokens/s and effective weight GB/s on B200.

Default workload: one single-token decode step of the Llama-2-110M-shaped Q8_0
matvec set (12 layers x {wq, wk, wv, wo 768x768, w1, w3 2048x768, w2 768x2048}
+ classifier 32000x768, 85 matvecs, batch 1), the Q8_0 int8 decode that the
"narray-llm" README measures.  Every matvec gets its own seeded N(0,1) x and
the set runs as one step: one q8_gemv_batched launch (each problem quantizes
its x to Q8_0 inside the kernel, then streams its weights).  The default run also reports the fused MoE
feed-forward step on its own workloads (moe_subrecords).

Other workloads (--workload): gemv_768, dense_ffn (--tokens 1|8),
llama2_110m_ffn (w1/w3 fused), moe_router (--tokens T), moe_layer
(--tokens 1|16), moe_30layer (--tokens 1|4|16|64|256).

Contract: ``python bench.py --gpus N --steps K --warmup W [--impl reference]``;
for N > 1 it is launched under torch.distributed.run, one rank per GPU, each
rank an independent replica of the step (weak scaling; the path has no
cross-GPU exchange).  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import math
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024
Q8_BLOCK_BYTES = 34  # per 32 weights


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama2_110m_q8_decode",
                    choices=["llama2_110m_q8_decode", "gemv_768", "dense_ffn", "llama2_110m_ffn",
                             "moe_router", "moe_layer",
                             "moe_30layer"])
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-subs", action="store_true",
                    help="skip the MoE sub-records of the default run")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="bound on the CPU baseline sample")
    ap.add_argument("--min-seconds", type=float, default=1.0,
                    help="timed work, in rounds of exactly --steps steps")
    return ap.parse_args()


def q8_bytes(rows, k):
    return rows * k // 32 * Q8_BLOCK_BYTES


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend):
        if self.world > 1:
            import datetime

            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        import torch
        t = torch.tensor([v], dtype=torch.float64,
                         device="cuda" if torch.cuda.is_available() else "cpu")
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def job_rate(dist, units_per_rank, local_ms):
    """Whole-job rate of N replicas: the units every rank processed over the
    slowest rank's device time (max over ranks).  Returns (rate per second,
    that time in ms)."""
    ms = dist.max(local_ms)
    return units_per_rank * dist.world / (ms / 1e3), ms


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
REASON_FIELDS = ["clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
                 "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]


class ClockSampler:
    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        q = "clocks.sm,clocks.max.sm,power.draw," + ",".join(REASON_FIELDS)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thr = threading.Thread(target=self._read, daemon=True)
        self.thr.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thr.join(timeout=2)
        try:
            err = self.proc.stderr.read()[-300:]
        except (OSError, ValueError):
            err = ""
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 3 + len(names):
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:]):
                if v.lower() == "active":
                    reasons.add(n)
        out = {"sm_mhz": statistics.median(sm) if sm else None,
               "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
               "samples": len(sm)}
        if not sm:
            out["sampler_output"] = (self.lines[:2], err.strip())
        return out


# ---------------------------------------------------------------------------
# in-graph event marks around the dominant kernel's launches
# ---------------------------------------------------------------------------
class Marks:
    """Records timing events as nodes of the graph being captured (external
    event records), so each replay times the marked launches on the device.
    The events are created (recorded once) before the capture starts."""

    def __init__(self, n_pairs: int):
        import torch
        self.events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                       for _ in range(n_pairs)]
        for a, b in self.events:
            a.record()
            b.record()
        self.used = 0

    @staticmethod
    def _rec(ev):
        import torch
        from cuda.bindings import runtime as rt
        err = rt.cudaEventRecordWithFlags(rt.cudaEvent_t(ev.cuda_event),
                                          rt.cudaStream_t(torch.cuda.current_stream().cuda_stream),
                                          rt.cudaEventRecordExternal)
        if int(err[0]) != 0:
            raise RuntimeError(f"cudaEventRecordWithFlags: {err}")

    def begin(self):
        self._rec(self.events[self.used][0])

    def end(self):
        self._rec(self.events[self.used][1])
        self.used += 1

    def ms(self):
        return [a.elapsed_time(b) for a, b in self.events[:self.used]]


class NoMarks:
    def begin(self):
        pass

    def end(self):
        pass


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
class LlamaDecode:
    """85 Q8_0 matvecs of one Llama-2-110M-shaped decode step, one batched launch."""
    name = "llama2_110m_q8_decode"
    kernel = "gemv_batched_kernel"

    def __init__(self, dev, tokens=None, gemv768=False, host_only=False):
        import torch

        from moe_up_gate_b200 import synth
        self.dev = dev
        self.host_only = host_only
        if gemv768:
            self.name = "gemv_768"
            mats = [("w", 768, 768)]
            seeds = [(synth.seed_of(1, 0, 0), synth.seed_of(1, 0, 1))]
        else:
            mats = synth.llama_matvec_set()
            seeds = []
            for i, (nm, rows, k) in enumerate(mats):
                layer, j = (i // 7, i % 7) if nm != "classifier" else (12, 0)
                seeds.append((synth.seed_of(2, layer, j), synth.seed_of(2, layer, j) + 500))
        self.mats = mats
        self.weight_bytes = sum(q8_bytes(r, k) for _, r, k in mats)
        # x: one fp32 buffer, each problem's x 16-byte aligned
        offs, o = [], 0
        for _, rows, k in mats:
            offs.append(o)
            o += k
        self.x_host = torch.empty(o, dtype=torch.float32)
        for (_, rows, k), off, (ws, xs) in zip(mats, offs, seeds):
            self.x_host[off:off + k] = synth.normal((1, k), xs)[0]
        self.w_fp32_seeds = seeds
        self.offs = offs
        self.weight_bytes = sum(q8_bytes(r, k) for _, r, k in mats)
        # L2 defeat: rotate through enough byte-identical weight copies
        self.copies = max(1, -(-3 * L2_BYTES // self.weight_bytes)) if self.weight_bytes > 4e6 else 1
        self.flush = self.weight_bytes < 4e6
        self.config = {"workload": self.name, "matvecs": len(mats), "batch": 1,
                       "weight_bytes_per_step": self.weight_bytes,
                       "l2": ("flush 256 MiB between steps" if self.flush else
                              f"{self.copies} rotating weight copies "
                              f"({self.copies * self.weight_bytes / 2**20:.0f} MiB)")}
        self.e2e_copies = ("every step: all matvec inputs host->device; the last matvec's "
                           "output (the classifier logits) device->host")
        if host_only:
            return
        from moe_up_gate_b200 import q8
        self.q8 = q8
        self.x_host = self.x_host.pin_memory()
        self.x = self.x_host.to(dev)
        self.y = [torch.empty((1, rows), dtype=torch.float32, device=dev) for _, rows, _ in mats]
        self.out_host = torch.empty(mats[-1][1], dtype=torch.float32).pin_memory()
        packed = []
        for (_, rows, k), (ws, _) in zip(mats, seeds):
            w = synth.normal((rows, k), ws, std=synth.W_STD, device=dev)
            packed.append(q8.pack(w))
            del w
        self.W = [packed]
        for c in range(1, self.copies):
            self.W.append([q8.Q8Tensor(P.qs.clone(), P.d.clone(), P.k, P.rows, P.n_mat, P.ld_d,
                                       P.mat_stride) for P in packed])
        self.sets = 1
        self.dominant_launches = 1
        self.tokens_per_step = 1
        self.launches_per_step = 1
        self.dominant_bytes = self.weight_bytes
        self.h2d_bytes = self.x_host.numel() * 4
        self.d2h_bytes = self.out_host.numel() * 4

    def issue(self, i, marks, input_set=None):
        W = self.W[i % self.copies]
        probs = [(Wm, self.x[off:off + Wm.k], y) for Wm, off, y in zip(W, self.offs, self.y)]
        marks.begin()
        self.q8.gemv_batched(probs, n_tok=1)
        marks.end()

    def unique_bytes(self, i):
        return self.weight_bytes

    def e2e_pre(self, i):
        self.x.copy_(self.x_host, non_blocking=True)

    def e2e_post(self, i):
        self.out_host.copy_(self.y[-1][0], non_blocking=True)

    # CPU oracle: one token of the same matvec set.  The weights are drawn
    # with the same seeds on self.dev (on "cpu" for the host-only reference
    # arm, where the values differ from a device draw but the recipe, shapes
    # and sizes are the same).
    def oracle_setup(self):
        import oracle
        from moe_up_gate_b200 import synth
        self.ow = []
        for (_, rows, k), (ws, _) in zip(self.mats, self.w_fp32_seeds):
            w = synth.normal((rows, k), ws, std=synth.W_STD, device=self.dev).cpu().numpy()
            self.ow.append(oracle.quantize_rows(w))
        self.ox = [self.x_host[o:o + k].numpy().reshape(1, k) for o, (_, _, k) in
                   zip(self.offs, self.mats)]

    def oracle_step(self):
        import oracle
        for (wq, wd), x in zip(self.ow, self.ox):
            xq, xd = oracle.quantize_rows(x)
            oracle.gemv(wq, wd, xq, xd)
        return 1  # tokens


ORACLE_TOKENS = 16


class MoeWorkload:
    """MoE (or dense) feed-forward layers through the public calls:
    quantize x -> group -> fused up/gate + SwiGLU (+ h quantization) -> down
    mul_mat_id -> combine (dense: quantize -> up/gate -> down GEMV; small
    dense batches: fp32 up/gate -> down GEMV on fp32 h, or, for h rows
    longer than the raw slot, h quantized once and the int8 down GEMV)

    layer_ids: the layers to build (default all; a parity test builds a few
    of them, with the same seeds and the same calls).  packed: the packed
    layers of another workload of the same kind and layers (their weights
    depend only on the layer's seed), reused instead of packing again.
    host_only: only the shapes, inputs and oracle side (the reference arm)."""
    kernel = "up_gate_kernel"

    def __init__(self, dev, kind, tokens, layer_ids=None, packed=None, host_only=False):
        import torch

        from moe_up_gate_b200 import synth
        self.dev = dev
        if kind == "dense_ffn":
            shape, layers, c, x_std = synth.DENSE_FFN, 1, 3, 1.0
        elif kind == "llama2_110m_ffn":
            # the Llama-2-110M feed-forward layers: w1 (gate) and w3 (up) are
            # separate weights, packed once into the combined up/gate tensor
            shape, layers, c, x_std = synth.LLAMA_FFN, synth.LLAMA_LAYERS, 2, 1.0
        elif kind == "moe_layer":
            shape, layers, c, x_std = synth.MOE_LAYER, 1, 4, 1.0
        else:
            shape, layers, c, x_std = synth.MOE_LAYER, synth.MOE_LAYERS, 5, synth.W_STD
        tokens = tokens or 1
        self.layer_ids = list(range(layers)) if layer_ids is None else list(layer_ids)
        self.name = kind
        self.c, self.x_std = c, x_std
        self.shape, self.layers, self.T = shape, len(self.layer_ids), tokens
        self.routed = shape.n_exp > 1
        U = shape.n_used
        D, F, E = shape.n_embd, shape.n_ff, shape.n_exp
        self.expert_bytes = q8_bytes(2 * F, D) + q8_bytes(D, F)
        layer_bytes = E * self.expert_bytes
        # L2 defeat: enough layer copies that a step never re-reads from L2
        per_step_max = self.layers * layer_bytes
        self.copies = 1 if per_step_max >= 3 * L2_BYTES else -(-3 * L2_BYTES // per_step_max)
        # rotating input sets: enough that the experts a set names were last
        # read more than 3x L2 of other weights ago (expected unique experts
        # of a step: E (1 - (1 - U/E)^T))
        uniq = E * (1 - (1 - U / E) ** tokens) if self.routed else 1
        self.sets = max(self.copies, 4 if self.routed else 1,
                        min(32, math.ceil(3 * L2_BYTES / (self.layers * uniq * self.expert_bytes)))
                        if self.routed else 1)
        # inputs per (set, layer)
        self.x_host, self.ids_host, self.p_host = [], [], []
        self.split = kind == "llama2_110m_ffn"
        for s in range(self.sets):
            xs, ids, ps = [], [], []
            for l in self.layer_ids:
                xs.append(synth.llama_ffn_tensors(l, tokens)["x"] if self.split and s == 0 else
                          synth.normal((tokens, D), synth.seed_of(c, l, 2) + 7919 * s, x_std))
                if self.routed:
                    ids.append(synth.routing_ids(tokens, E, U, synth.seed_of(c, l, 3) + 7919 * s))
                    ps.append(synth.routing_weights(tokens, U, synth.seed_of(c, l, 4) + 7919 * s))
            self.x_host.append(torch.stack(xs))
            if self.routed:
                self.ids_host.append(torch.stack(ids))
                self.p_host.append(torch.stack(ps))
        Uu = U if self.routed else 1
        P = tokens * Uu
        # algorithmic bytes: the experts each layer's ids actually name
        self.step_bytes, self.up_gate_bytes = [], []
        self.fused = self.routed and P <= 32 and D <= 4096 and F <= 2048
        for s in range(self.sets):
            tot, ug = 0, 0
            for li in range(self.layers):
                ne = len(set(self.ids_host[s][li].flatten().tolist())) if self.routed else 1
                tot += ne * self.expert_bytes
                ug += ne * q8_bytes(2 * F, D)
            self.step_bytes.append(tot)
            # bytes of one launch of the dominant kernel (a layer's up/gate, or
            # the whole layer when it is fused)
            self.up_gate_bytes.append((tot if self.fused else ug) / self.layers)
        self.tokens_per_step = tokens
        # the paths q8_moe_ffn takes: the fp32 calls for dense batches up to
        # 1024 rows and routed batches up to 32 pairs (the fused kernel
        # when it applies); larger routed batches group once (tensor cores
        # for the experts with at least 4 rows)
        self.small = P <= 1024 and E <= 512 and (not self.routed or P <= 32)
        self.config = {"workload": kind, "tokens": tokens, "layers": self.layers, "n_embd": D,
                       "n_ff": F, "n_experts": E, "n_used": Uu,
                       "mean_weight_bytes_per_step": statistics.mean(self.step_bytes),
                       "l2": (f"{self.copies} rotating weight copies, {self.sets} input sets"
                              if self.copies > 1 else
                              f"weights per step > 3x L2; {self.sets} input sets")}
        self.e2e_copies = ("every step: x (and ids, routing weights) host->device; every "
                           "layer's output device->host")
        if host_only:
            return
        from moe_up_gate_b200 import q8
        self.q8 = q8
        if packed is not None:
            self.L = packed
        elif self.split:
            self.L = []
            for l in self.layer_ids:
                t = synth.llama_ffn_tensors(l, 1, device=dev)
                self.L.append((q8.pack_up_gate(t["w1"], t["w3"]), q8.pack(t["w2"])))
                del t
        else:
            self.L = []
            for l in self.layer_ids:
                t = synth.moe_layer_tensors(c, l, shape, 1, x_std, device=dev)
                UG = q8.pack(t["up_gate"])
                DN = q8.pack(t["down"])
                del t
                self.L.append((UG, DN))
        torch.cuda.synchronize()
        self.Lc = [self.L]
        for cc in range(1, self.copies):
            self.Lc.append([tuple(q8.Q8Tensor(P_.qs.clone(), P_.d.clone(), P_.k, P_.rows,
                                              P_.n_mat, P_.ld_d, P_.mat_stride) for P_ in pair)
                            for pair in self.L])
        self.x_host = [xh.pin_memory() for xh in self.x_host]
        self.ids_host = [ih.pin_memory() for ih in self.ids_host]
        self.p_host = [ph.pin_memory() for ph in self.p_host]
        self.x = [xh.to(dev) for xh in self.x_host]
        self.ids = [ih.to(dev) for ih in self.ids_host]
        self.p = [ph.to(dev) for ph in self.p_host]
        self.ws = q8.moe_workspace(tokens, Uu, E, dev) if self.routed else None
        self.xq = torch.empty((tokens, D), dtype=torch.int8, device=dev)
        self.xd = torch.empty((tokens, D // 32), dtype=torch.float16, device=dev)
        self.h = torch.empty((P, F), dtype=torch.float32, device=dev)
        self.hq = torch.empty((P, F), dtype=torch.int8, device=dev)
        self.hd = torch.empty((P, F // 32), dtype=torch.float16, device=dev)
        # dense h rows longer than the 16 KB raw slot of the streaming
        # kernels are quantized once before the down GEMV
        self.h_once = not self.routed and F * 4 > 16 * 1024
        self.y = torch.empty((tokens, Uu, D), dtype=torch.float32, device=dev)
        self.out = torch.empty((self.layers, tokens, D), dtype=torch.float32, device=dev)
        self.out_host = torch.empty((self.layers, tokens, D), dtype=torch.float32).pin_memory()
        # routed batches of at most 32 pairs: q8_moe_ffn runs the whole layer
        # as one kernel (the dominant kernel is then the layer kernel)
        if self.fused:
            self.kernel = "moe_layer_kernel"
            self.ffn_ws = q8.moe_ffn_workspace(tokens, U, E, D, F, dev)
            self.launches_per_step = self.layers
        elif self.small:
            self.launches_per_step = self.layers * (3 if self.routed or self.h_once else 2)
        elif self.routed:
            # quantize x, group, up/gate (dp4a + tensor cores), quantize h,
            # down (dp4a + tensor cores), combine; the timed unit is the
            # up/gate step: tc_kernel for the experts with >= 4 rows and
            # up_gate_kernel for the rest
            self.kernel = "up_gate_step"
            self.launches_per_step = self.layers * 8
        else:
            self.launches_per_step = self.layers * 4
        self.dominant_launches = self.layers
        self.h2d_bytes = self.x_host[0].numel() * 4 + (
            (self.ids_host[0].numel() * 4 + self.p_host[0].numel() * 4) if self.routed else 0)
        self.d2h_bytes = self.out_host.numel() * 4

    def issue(self, i, marks, input_set=None):
        q8 = self.q8
        s = i % self.sets if input_set is None else input_set
        layers = self.Lc[i % self.copies]
        T = self.T
        if self.fused:
            # the public whole-step call: one fused kernel per layer
            for l, (UG, DN) in enumerate(layers):
                marks.begin()
                q8.moe_ffn(UG, DN, self.x[s][l], self.ids[s][l], self.p[s][l], ws=self.ffn_ws,
                           out=self.out[l])
                marks.end()
            return
        if self.small:
            # small batches: the fp32 calls (x and h quantized inside the
            # kernels, routing grouped in every CTA), the same kernels
            # q8_moe_ffn runs: routed 3 launches per layer, dense 2 (3 when
            # h is quantized once)
            for l, (UG, DN) in enumerate(layers):
                x = self.x[s][l]
                if self.routed:
                    ids = self.ids[s][l]
                    marks.begin()
                    q8.moe_up_gate_swiglu_fp32(UG, x, ids, h=self.h)
                    marks.end()
                    q8.mul_mat_id_fp32(DN, self.h, ids, True, y=self.y)
                    q8.moe_combine(self.y, self.p[s][l], out=self.out[l])
                else:
                    marks.begin()
                    q8.moe_up_gate_swiglu_fp32(UG, x, None, h=self.h)
                    marks.end()
                    if self.h_once:
                        # h rows longer than a CTA's raw slot: h quantized
                        # once, then the Q8_0 GEMV (as q8_moe_ffn does)
                        q8._call("q8_quantize_row", q8._ptr(self.h), T, self.h.shape[1],
                                 q8._ptr(self.hq), q8._ptr(self.hd), q8._stream())
                        q8.gemv(DN, self.hq, self.hd, y=self.out[l])
                    else:
                        q8.gemv_batched([(DN, self.h, self.out[l])], n_tok=T)
            return
        for l, (UG, DN) in enumerate(layers):
            x = self.x[s][l]
            q8._call("q8_quantize_row", q8._ptr(x), T, UG.k, q8._ptr(self.xq), q8._ptr(self.xd),
                     q8._stream())
            if self.routed:
                U = self.shape.n_used
                q8.moe_group(self.ids[s][l], UG.n_mat, ws=self.ws)
                marks.begin()
                q8.moe_up_gate_swiglu_pregrouped(UG, self.xq, self.xd, U, self.ws, self.h, self.hq,
                                                 self.hd)
                marks.end()
                q8.mul_mat_id_pregrouped(DN, self.hq, self.hd, T, U, True, self.ws, self.y)
                q8.moe_combine(self.y, self.p[s][l], out=self.out[l])
            else:
                marks.begin()
                q8._call("q8_moe_up_gate_swiglu", q8.ctypes.byref(UG.c()), q8._ptr(self.xq),
                         q8._ptr(self.xd), T, None, 1, q8._ptr(self.h), q8._ptr(self.hq),
                         q8._ptr(self.hd), None, None, None, 0, q8._stream())
                marks.end()
                q8.gemv(DN, self.hq, self.hd, y=self.out[l])

    def unique_bytes(self, i):
        return self.step_bytes[i % self.sets]

    def dominant_bytes_at(self, i):
        return self.up_gate_bytes[i % self.sets]

    def e2e_pre(self, i):
        s = i % self.sets
        self.x[s].copy_(self.x_host[s], non_blocking=True)
        if self.routed:
            self.ids[s].copy_(self.ids_host[s], non_blocking=True)
            self.p[s].copy_(self.p_host[s], non_blocking=True)

    def e2e_post(self, i):
        self.out_host.copy_(self.out, non_blocking=True)

    def oracle_setup(self):
        import oracle
        from moe_up_gate_b200 import synth
        # one layer through the oracle (its own quantization of the fp32
        # weights, drawn with the layer's seeds on self.dev)
        import numpy as np
        l0 = self.layer_ids[0]
        if self.split:
            t = synth.llama_ffn_tensors(l0, 1, device=self.dev)
            g, u = oracle.quantize_rows(t["w1"].cpu().numpy()), oracle.quantize_rows(
                t["w3"].cpu().numpy())
            # the oracle's moe_ffn on the row concatenation [w1; w3] is its
            # separate-weights path, bit for bit (pinned)
            self.o_ug = (np.concatenate([g[0], u[0]]), np.concatenate([g[1], u[1]]))
            self.o_dn = oracle.quantize_rows(t["w2"].cpu().numpy())
        else:
            t = synth.moe_layer_tensors(self.c, l0, self.shape, 1, self.x_std, device=self.dev)
            self.o_ug = oracle.quantize_rows(t["up_gate"].cpu().numpy())
            self.o_dn = oracle.quantize_rows(t["down"].cpu().numpy())
        # a bounded sample: at most ORACLE_TOKENS of the step's tokens per
        # oracle step (the oracle's time grows with the tokens)
        self.o_tok = min(self.T, ORACLE_TOKENS)
        self.o_x = self.x_host[0][0][:self.o_tok].numpy()
        self.o_ids = self.ids_host[0][0][:self.o_tok].numpy() if self.routed else None
        self.o_p = self.p_host[0][0][:self.o_tok].numpy() if self.routed else None

    def oracle_step(self):
        import oracle
        oracle.moe_ffn(self.o_ug[0], self.o_ug[1], self.o_dn[0], self.o_dn[1], self.o_x,
                       self.o_ids, self.o_p)
        return self.o_tok / self.layers  # one layer of a layers-deep step


class RouterWorkload:
    """The router before the MoE layer (q8_route): fp32 router weights
    [128, 2816] and T tokens' x -> top-8 ids and routing weights, one launch
    per step.  The bytes that must be read are the router weights (fp32) and
    the tokens' x."""
    kernel = "route_kernel"

    def __init__(self, dev, tokens, host_only=False):
        import torch

        from moe_up_gate_b200 import synth
        shape = synth.MOE_LAYER
        self.dev, self.T, self.name = dev, tokens or 1, "moe_router"
        self.D, self.E, self.U = shape.n_embd, shape.n_exp, shape.n_used
        self.w_bytes = self.E * self.D * 4
        self.copies = max(1, -(-3 * L2_BYTES // self.w_bytes))
        self.sets, self.flush, self.layers = 1, False, 1
        self.w_seed = synth.seed_of(6, 0, 0)
        self.x_host = synth.normal((self.T, self.D), synth.seed_of(6, 0, 1))
        self.tokens_per_step = self.T
        self.step_bytes = self.w_bytes + self.T * self.D * 4
        self.config = {"workload": self.name, "tokens": self.T, "n_embd": self.D,
                       "n_experts": self.E, "n_used": self.U,
                       "weight_bytes_per_step": self.w_bytes,
                       "l2": f"{self.copies} rotating router-weight copies"}
        self.e2e_copies = "every step: x host->device; ids and routing weights device->host"
        if host_only:
            return
        from moe_up_gate_b200 import q8
        self.q8 = q8
        w = synth.normal((self.E, self.D), self.w_seed, synth.W_STD, device=dev)
        self.W = [w] + [w.clone() for _ in range(self.copies - 1)]
        self.x_host = self.x_host.pin_memory()
        self.x = self.x_host.to(dev)
        self.ids = torch.empty((self.T, self.U), dtype=torch.int32, device=dev)
        self.rw = torch.empty((self.T, self.U), dtype=torch.float32, device=dev)
        self.ids_host = torch.empty_like(self.ids, device="cpu").pin_memory()
        self.rw_host = torch.empty_like(self.rw, device="cpu").pin_memory()
        self.launches_per_step = self.dominant_launches = 1
        self.h2d_bytes = self.x_host.numel() * 4
        self.d2h_bytes = self.ids.numel() * 4 + self.rw.numel() * 4

    def issue(self, i, marks, input_set=None):
        marks.begin()
        self.q8.route(self.W[i % self.copies], self.x, self.U, ids=self.ids, route_w=self.rw)
        marks.end()

    def unique_bytes(self, i):
        return self.step_bytes

    def dominant_bytes_at(self, i):
        return self.step_bytes

    def e2e_pre(self, i):
        self.x.copy_(self.x_host, non_blocking=True)

    def e2e_post(self, i):
        self.ids_host.copy_(self.ids, non_blocking=True)
        self.rw_host.copy_(self.rw, non_blocking=True)

    def oracle_setup(self):
        from moe_up_gate_b200 import synth
        self.o_w = synth.normal((self.E, self.D), self.w_seed, synth.W_STD,
                                device=self.dev).cpu().numpy()
        self.o_tok = min(self.T, ORACLE_TOKENS)
        self.o_x = self.x_host[:self.o_tok].numpy()
        self.layers = 1

    def oracle_step(self):
        import oracle
        oracle.route(oracle.router_logits(self.o_w, self.o_x), self.U)
        return self.o_tok


def make_workload(workload, tokens, dev, host_only=False, packed=None):
    if workload == "moe_router":
        return RouterWorkload(dev, tokens, host_only=host_only)
    if workload == "llama2_110m_q8_decode":
        return LlamaDecode(dev, host_only=host_only)
    if workload == "gemv_768":
        return LlamaDecode(dev, gemv768=True, host_only=host_only)
    return MoeWorkload(dev, workload, tokens, packed=packed, host_only=host_only)


# ---------------------------------------------------------------------------
# traffic counters recorded by ncu (profiles/traffic.json), valid only for
# the kernel sources they were taken on
# ---------------------------------------------------------------------------
def gpu_id(local_rank: int) -> str:
    """nvidia-smi --id for this rank's device (PCI bus id when torch knows it)."""
    import torch
    try:
        pr = torch.cuda.get_device_properties(local_rank)
        return f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
    except (AttributeError, RuntimeError, TypeError, ValueError):
        return str(local_rank)


# the sources each kernel is built from (its traffic record is void once any
# of them changes)
KERNEL_SOURCES = {
    "gemv_batched_kernel": ["q8_matmul.cu"],
    "route_kernel": ["q8_route.cu"],
    "up_gate_kernel": ["q8_moe.cu"],
    "moe_layer_kernel": ["q8_layer.cu"],
    "tc_kernel": ["q8_tc.cu", "q8_tc.cuh"],
    "up_gate_step": ["q8_moe.cu", "q8_tc.cu", "q8_tc.cuh"],
}
SHARED_SOURCES = ["q8_stream.cuh", "q8_device.cuh", "q8_ptx.cuh", "q8_internal.h"]


def kernel_source_hash(kernel=None):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "moe_up_gate_b200", "csrc")
    files = (sorted(os.listdir(csrc)) if kernel not in KERNEL_SOURCES else
             sorted(KERNEL_SOURCES[kernel] + SHARED_SOURCES))
    for fn in files:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, kernel):
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    ent = rec.get(f"{workload}:{kernel}")
    if not ent or ent.get("source_hash") != kernel_source_hash(kernel):
        return None
    return ent.get("dram_bytes_per_launch")


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, ValueError, KeyError):
        return 6650.0, "fallback"


# ---------------------------------------------------------------------------
# CPU oracle timing
# ---------------------------------------------------------------------------
def time_oracle(wl, seconds, steps=None):
    import oracle
    wl.oracle_setup()
    cores = oracle.max_threads()
    done, t0, n = 0.0, time.perf_counter(), 0
    times = []
    while True:
        a = time.perf_counter()
        done += wl.oracle_step()
        times.append(time.perf_counter() - a)
        n += 1
        if steps is not None:
            if n >= steps:
                break
        elif time.perf_counter() - t0 >= seconds:
            break
    return done, sum(times), n, cores, times


# ---------------------------------------------------------------------------
def run_reference(args, dist):
    """The reference arm: the CPU oracle, as it stands, on the host cores.
    Host only: the inputs are drawn on the CPU with the workload's seeds, and
    nothing of the CUDA library is loaded."""
    if dist.rank != 0:
        return
    import oracle
    wl = make_workload(args.workload, args.tokens, "cpu", host_only=True)
    wl.oracle_setup()
    for _ in range(args.warmup):
        wl.oracle_step()
    t0 = time.perf_counter()
    toks = 0.0
    for _ in range(args.steps):
        toks += wl.oracle_step()
    el = time.perf_counter() - t0
    v = toks / el
    sample = (f"{args.steps} steps of one {wl.name} token through the scalar C oracle "
              f"(inputs drawn on the CPU with the workload's seeds)"
              if isinstance(wl, LlamaDecode) else
              f"{args.steps} x one layer of {wl.name} (T={wl.T}; the first {wl.o_tok} tokens) "
              f"through the scalar C oracle, counted as 1/{wl.layers} of a step (inputs drawn "
              f"on the CPU with the workload's seeds)")
    out = {"metric": METRIC, "value": v, "unit": "tokens/s", "impl": "reference",
           "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "int8 x int8 -> int32, fp64 sums",
           "data": DATA, "config": dict(wl.config, parallelism=f"replicas x{dist.world}"),
           "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": oracle.max_threads(),
                            "kind": "oracle", "sample": sample},
           "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out))


METRIC = "Q8_0 decode tokens/s"
DATA = "synthetic (seeded N(0, 0.02) weights quantized to Q8_0, N(0,1) inputs)"

# The default run reports, beside the headline decode step, the fused MoE
# feed-forward step on these workloads (one sub-record each).
SUB_WORKLOADS = [("moe_layer", 1), ("moe_30layer", 1), ("moe_30layer", 256)]


def measure(wl, args, dist, stream, cpu_seconds):
    """Time K steps of workload wl (device events), its dominant kernel
    (in-graph event marks), the end-to-end rate through host buffers and the
    oracle on the host cores.  Returns the record (without the shared keys)."""
    import torch
    K, W = args.steps, max(args.warmup, 3)
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device=wl.dev) \
        if getattr(wl, "flush", False) else None

    # CUDA graphs without timing marks for the step rate: one per warm-up
    # step, and the K timed steps in one graph (back to back on the device,
    # no host replay between steps) unless an L2 flush must run between
    # them (then one graph per step); and one graph per timed step with
    # event marks around the dominant launches (the kernel time), kept out of
    # the step-rate graphs
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        wl.issue(0, NoMarks())  # eager warm-up (sets kernel attributes)
    torch.cuda.synchronize()

    def capture(i, m, input_set=None, n_steps=1):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for j in range(i, i + n_steps):
                wl.issue(j, m, input_set)
        return g

    graphs = [capture(i, NoMarks()) for i in range(W + (K if flush is not None else 0))]
    timed_graph = capture(W, NoMarks(), n_steps=K) if flush is None else None
    marks = [Marks(wl.dominant_launches) for _ in range(K)]
    mgraphs = [capture(W + i, marks[i]) for i in range(K)]
    torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        for i in range(W):
            if flush is not None:
                flush.zero_()
            graphs[i].replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_id(dist.local))
    clocks.start()
    time.sleep(0.5)  # let the sampler start before the timed work

    ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    st_ev = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    en_ev = [torch.cuda.Event(enable_timing=True) for _ in range(K)]

    def timed_steps(step, all_steps=None):
        """K steps, bracketed by a barrier + synchronize on both sides; ms of
        device time, max over ranks.  Timed by one pair of events around the K
        steps (all_steps() issues them at once when given, else step(i) each),
        or, when an L2 flush runs between steps, by a pair around each step
        (the flush stays outside the timed intervals)."""
        torch.cuda.synchronize()
        dist.barrier()
        with torch.cuda.stream(stream):
            if flush is None:
                ev[0].record(stream)
                if all_steps is not None:
                    all_steps()
                else:
                    for i in range(K):
                        step(i)
                ev[1].record(stream)
            else:
                for i in range(K):
                    flush.zero_()
                    st_ev[i].record(stream)
                    step(i)
                    en_ev[i].record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        ms = (ev[0].elapsed_time(ev[1]) if flush is None else
              sum(a.elapsed_time(b) for a, b in zip(st_ev, en_ev)))
        return dist.max(ms)

    def one_round():
        if timed_graph is not None:
            return timed_steps(None, all_steps=timed_graph.replay)
        return timed_steps(lambda i: graphs[W + i].replay())

    torch.cuda.nvtx.range_push("timed")
    first_ms = one_round()
    rounds = int(min(1000, max(3, math.ceil(args.min_seconds * 1e3 / max(first_ms, 1e-3)))))
    round_ms = [first_ms] + [one_round() for _ in range(rounds - 1)]
    torch.cuda.nvtx.range_pop()
    # the dominant kernel: the same steps with the in-graph marks
    dom_ms = []
    for _ in range(max(3, min(rounds, 50))):
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            for i in range(K):
                if flush is not None:
                    flush.zero_()
                mgraphs[i].replay()
        torch.cuda.synchronize()
        for m in marks:
            dom_ms.extend(m.ms())
    clk = clocks.stop()
    total_ms = statistics.median(round_ms)

    # end to end through the public API with host buffers: every step copies
    # its inputs from pinned host memory, runs the step (graphs of the same
    # public calls, on the same rotation of weight copies and input sets, with
    # the same L2 flush) and copies its result back
    n_e2e = max(wl.copies, wl.sets)
    e2e_graphs = [capture(c, NoMarks(), c % wl.sets) for c in range(n_e2e)]

    def e2e_step(i):
        wl.e2e_pre(i)
        e2e_graphs[i % n_e2e].replay()
        wl.e2e_post(i)

    e2e_ms = timed_steps(e2e_step)
    e2e_rate, _ = job_rate(dist, wl.tokens_per_step * K, e2e_ms)

    n = dist.world
    value, total_ms = job_rate(dist, wl.tokens_per_step * K, total_ms)
    step_bytes = statistics.mean(wl.unique_bytes(W + i) for i in range(K))
    peak, peak_kind = measured_peak()
    if isinstance(wl, LlamaDecode):
        dom_bytes = wl.dominant_bytes
    else:
        dom_bytes = statistics.mean(wl.dominant_bytes_at(W + i) for i in range(K))
    marked_ms = statistics.mean(dom_ms) if dom_ms else None
    if wl.launches_per_step == wl.dominant_launches:
        # the step is the dominant kernel's launches alone: the timed rounds
        # bracket exactly K x those launches with one event pair, an upper
        # bound of their average duration (back-to-back launches, no marks)
        dom_avg_ms = total_ms / (K * wl.dominant_launches)
        dom_timer = ("timed rounds: each step is only these launches; round time / launches")
    else:
        dom_avg_ms = marked_ms
        dom_timer = ("event-record nodes around the kernel's launches inside the step graphs "
                     "(they include the marked launches' own launch latency)")
    achieved = dom_bytes / (dom_avg_ms / 1e3) / 1e9 if dom_avg_ms else None
    traffic = recorded_traffic(wl.name + (f"_t{wl.T}" if hasattr(wl, "T") else ""), wl.kernel)
    out = {
        "value": value, "unit": "tokens/s", "ms_per_step": total_ms / K,
        "config": dict(wl.config, parallelism=f"replicas x{n}"),
        "timing": {"rounds": len(round_ms),
                   "round_ms_min_median_max": [min(round_ms), total_ms, max(round_ms)],
                   "step_timer": ("one event pair around each round of K steps (the K steps "
                                  "replayed as one CUDA graph)"
                                  if flush is None else
                                  "an event pair around each step (the L2 flush between "
                                  "steps is not timed)")},
        "effective_weight_GBps": step_bytes / (total_ms / K / 1e3) / 1e9,
        "effective_weight_frac_of_hbm": step_bytes / (total_ms / K / 1e3) / 1e9 / peak,
        "roofline": {"bound": "hbm", "kernel": wl.kernel, "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": (achieved / peak) if achieved else None,
                     "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                     "bytes_per_launch": dom_bytes, "avg_launch_ms": dom_avg_ms,
                     "launch_timer": dom_timer, "marked_launch_ms": marked_ms,
                     "launches_marked": len(dom_ms), "traffic": traffic},
        "clocks": clk,
        "e2e": {"value": e2e_rate, "unit": "tokens/s",
                "h2d_bytes_per_step": wl.h2d_bytes, "d2h_bytes_per_step": wl.d2h_bytes,
                "copies": wl.e2e_copies},
        "gpu_launches": wl.launches_per_step * K,
    }
    if dist.rank == 0 and n == 1 and cpu_seconds > 0:
        done, el, nsteps, cores, _ = time_oracle(wl, cpu_seconds)
        out["cpu_baseline"] = {
            "value": done / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": (f"{nsteps} tokens of {wl.name} through the scalar C oracle "
                       f"(OpenMP over output rows), {el:.1f} s"
                       if isinstance(wl, LlamaDecode) else
                       f"{nsteps} x one layer of {wl.name} (T={wl.T}) through the scalar C "
                       f"oracle (the first {wl.o_tok} of its tokens), counted as "
                       f"1/{wl.layers} of a step, {el:.1f} s")}
    del graphs, timed_graph, mgraphs, e2e_graphs
    return out


def main():
    args = parse()
    dist = Dist()
    if args.impl == "reference":
        run_reference(args, dist)
        return
    import torch
    torch.cuda.set_device(dist.local)
    dev = f"cuda:{dist.local}"
    dist.init("nccl")
    from moe_up_gate_b200 import q8
    q8.load()
    stream = torch.cuda.Stream(device=dev)
    cpu_s = 0.0 if args.no_cpu_baseline else args.cpu_seconds
    wl = make_workload(args.workload, args.tokens, dev)
    rec = measure(wl, args, dist, stream, cpu_s)
    del wl
    out = {"metric": METRIC, "value": rec.pop("value"), "unit": rec.pop("unit"),
           "n_gpus": dist.world, "steps": args.steps, "warmup": max(args.warmup, 3),
           "ms_per_step": rec.pop("ms_per_step"), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "int8 x int8 -> int32, fp32 sums", "data": DATA}
    out.update(rec)
    if args.workload == "llama2_110m_q8_decode" and not args.no_subs:
        # the fused MoE feed-forward step (the subject op) on its own workloads
        subs, packed30 = [], None
        for name, T in SUB_WORKLOADS:
            torch.cuda.empty_cache()
            w = make_workload(name, T, dev, packed=packed30 if name == "moe_30layer" else None)
            if name == "moe_30layer":
                packed30 = w.L
            r = measure(w, args, dist, stream, cpu_s / 3)
            r["workload"] = f"{name}_t{T}"
            subs.append(r)
            del w
        out["moe_subrecords"] = subs
    if dist.rank == 0:
        print(json.dumps(out))
    dist.close()


if __name__ == "__main__":
    main()
