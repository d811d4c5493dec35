#!/usr/bin/env python
"""Decode benchmark on B200: decoded fp16 GB/s and fraction of the HBM roofline.

One step = one pass of every decode workload over its synthetic input:
  C1  INT4 group dequant, 1,048,576 codes, group 256
  C2  INT8 per-row dequant, 8192 x 8192
  C3  zero-run decode, 8 x 2048 x 11008 fp16 ReLU-like activations
  C4  fused LZ4 -> INT4 -> fp16, 4096 x 14336, group 128, 64 KB blocks
  C4u INT4 group dequant of C4's matrix without the LZ4 layer (the
      uncompressed variant at the large shape, 4096 x 14336, group 128)
  C5  8 Llama-2-70B-shaped layers (q, o, k, v, gate, up, down), fused LZ4 ->
      INT4 -> fp16: one index launch over the blocks of all layers, then each
      layer expanded (one launch) into one reused buffer
The headline value is the step's total decoded fp16 bytes / step time
(GB/s, 1e9). Inputs are resident in HBM when the timed region starts; the
step touches ~16 GB, far more than L2, so no L2 flush is needed between
steps. Per-codec figures and the roofline fraction of the dominant kernel
(the fused LZ4 decode of C5) are reported beside it.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lt|reference]
Under torchrun each rank decodes its own copy of the workload (weak scaling,
no data-path collective); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decoded FP16 GB/s per codec; % of B200 HBM roofline (bytes read+written)"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0

# dram__bytes_read.sum + dram__bytes_write.sum of one C5 layer's decode (its
# expand launch + 1/8 of the all-layer index launch), from the ncu capture
# summarised under profiles/; valid only while the kernel sources hash to
# `sources_sha256`.
NCU_TRAFFIC = {"sources_sha256": "c85327e5cd2e969ba9fdc33d53b18f44d0ee3e110f7335c723bdecc7e43fea6a", "bytes_per_launch": 2355703808,
               "profile": "profiles/k_lz4_c5_layer_traffic.md"}


def kernel_sources_sha() -> str:
    h = hashlib.sha256()
    for f in ("lt_lz4.cu", "lt_common.cuh"):
        with open(os.path.join(ROOT, "weight_dequantization_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["lt", "reference"], default="lt")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=8, help="C5 layers (8 is the workload)")
    ap.add_argument("--gemm-shapes", default="q/o,k/v,gate/up,down",
                    help="C5 weight shapes of the GEMM leg (G): comma-separated subset of q/o, k/v, gate/up, down")
    ap.add_argument("--gemm-m", default="1,16,128,4096", help="batch sizes M of the GEMM leg (G)")
    ap.add_argument("--no-parity", action="store_true",
                    help="skip the parity pass (profiling runs only: the line then says parity was not checked)")
    ap.add_argument("--only", default="C1,C2,C3,C4,C4u,C5,V,S,G",
                    help="comma-separated subset of the workloads to run (profiling); the bench line uses all. "
                         "C1-C5 form the timed step; V (value-dictionary decode), S (the streaming API over "
                         "the C5 layers) and G (fused decode -> GEMM on the C5 shapes) are timed on their own "
                         "afterwards")
    return ap.parse_args()


# ----------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def dist_init(world):
    if world <= 1:
        return None
    import datetime

    import torch.distributed as dist

    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, dist) -> float:
    from weight_dequantization_b200.shard import reduce_max

    return reduce_max(x, device="cuda") if dist is not None else x


def sum_over_ranks(x: float, dist) -> float:
    from weight_dequantization_b200.shard import reduce_sum

    return reduce_sum(x, device="cuda") if dist is not None else x


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.rows = []
        self.proc = None
        self.gpu_id = gpu_id

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 7:
                self.rows.append(parts)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, smax, reasons = [], [], set()
        for r in self.rows:
            try:
                sm.append(float(r[0]))
                smax.append(float(r[1]))
            except ValueError:
                continue
            for i, nm in enumerate(names):
                if r[3 + i].lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_id_for(dev_index: int) -> str:
    import torch

    try:
        u = str(torch.cuda.get_device_properties(dev_index).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        return vis.split(",")[dev_index] if vis else str(dev_index)


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

STEP_CODECS = ("C1", "C2", "C3", "C4", "C4u")  # single-call units of a step, in order; then C5


def build_host_workload(rank: int, layers: int, only=("C1", "C2", "C3", "C4", "C4u", "C5")):
    """Seeded host inputs; each rank gets its own seeds (weak scaling)."""
    from weight_dequantization_b200.synth import workloads as W

    off = 1000 * rank
    make = {
        "C1": lambda: W.c1_int4(seed=1 + off),
        "C2": lambda: W.c2_int8(seed=2 + off),
        "C3": lambda: W.c3_zrle(seed=3 + off),
        "C4": lambda: W.c4_lz4_int4(seed=4 + off, keep_packed="C4u" in only),
        "C5": lambda: W.c5_layers(layers=layers, seed=5 + off),
    }
    hw = {k: make[k]() for k in ("C1", "C2", "C3", "C4", "C5") if k in only or (k == "C4" and "C4u" in only)}
    if "C4u" in only:
        # the same matrix, codes, scales and zero points as C4, not compressed
        c4 = hw["C4"]
        hw["C4u"] = dict(kind="int4", rows=c4["rows"], cols=c4["cols"], group_size=c4["group_size"],
                         packed=c4.pop("packed"), scales=c4["scales"], zeros=c4["zeros"])
        if "C4" not in only:
            del hw["C4"]
    return hw


def nbytes(a) -> int:
    return 0 if a is None else int(a.nbytes)


def algorithmic_bytes(hw):
    """Bytes the method must read + write per codec (actual buffers)."""
    out = {}
    if "C1" in hw:
        c1 = hw["C1"]
        out["C1"] = (nbytes(c1["packed"]) + nbytes(c1["scales"]) + nbytes(c1["zeros"]), 2 * c1["rows"] * c1["cols"])
    if "C2" in hw:
        c2 = hw["C2"]
        out["C2"] = (nbytes(c2["q"]) + nbytes(c2["scales"]) + nbytes(c2["zeros"]), 2 * c2["rows"] * c2["cols"])
    if "C3" in hw:
        c3 = hw["C3"]
        out["C3"] = (nbytes(c3["enc"]) + nbytes(c3["offsets"]), 2 * c3["n"])
    if "C4" in hw:
        c4 = hw["C4"]
        out["C4"] = (nbytes(c4["comp"]) + nbytes(c4["offsets"]) + nbytes(c4["scales"]) + nbytes(c4["zeros"]),
                     2 * c4["rows"] * c4["cols"])
    if "C4u" in hw:
        c = hw["C4u"]
        out["C4u"] = (nbytes(c["packed"]) + nbytes(c["scales"]) + nbytes(c["zeros"]), 2 * c["rows"] * c["cols"])
    layer = []
    if "C5" in hw:
        for mats in hw["C5"]:
            rd = sum(nbytes(m["comp"]) + nbytes(m["offsets"]) + nbytes(m["scales"]) + nbytes(m["zeros"])
                     for m in mats)
            wr = sum(2 * m["rows"] * m["cols"] for m in mats)
            layer.append((rd, wr))
        out["C5"] = (sum(r for r, _ in layer), sum(w for _, w in layer))
    return out, layer


class DeviceWorkload:
    """Device copies of the inputs, output buffers, and pinned host staging
    buffers for the end-to-end measurement."""

    def __init__(self, hw, pinned: bool):
        import numpy as np
        import torch

        self.torch = torch
        self.hw = hw
        self.h2d = []  # (pinned host tensor, device tensor)
        self.unit_h2d = {}  # unit ("C1", ..., ("C5", layer)) -> its (pinned host, device) pairs
        unit = [None]

        def put(a):
            if a is None:
                return None
            a = np.ascontiguousarray(a)
            if a.dtype == np.uint16:
                a = a.view(np.int16)
            elif a.dtype == np.uint64:
                a = a.view(np.int64)
            host = torch.from_numpy(a)
            d = host.to("cuda")
            if pinned:
                ph = torch.empty_like(host).pin_memory()
                ph.copy_(host)
                self.h2d.append((ph, d))
                self.unit_h2d.setdefault(unit[0], []).append((ph, d))
            return d

        if "C1" in hw:
            c1 = hw["C1"]
            unit[0] = "C1"
            self.c1 = dict(packed=put(c1["packed"]), scales=put(c1["scales"]), zeros=put(c1["zeros"]))
            self.c1_out = torch.empty(c1["rows"] * c1["cols"], dtype=torch.float16, device="cuda")
        if "C2" in hw:
            c2 = hw["C2"]
            unit[0] = "C2"
            self.c2 = dict(q=put(c2["q"]), scales=put(c2["scales"]))
            self.c2_out = torch.empty(c2["rows"] * c2["cols"], dtype=torch.float16, device="cuda")
        if "C3" in hw:
            c3 = hw["C3"]
            unit[0] = "C3"
            self.c3 = dict(enc=put(c3["enc"]), offsets=put(c3["offsets"]))
            self.c3_out = torch.empty(c3["n"], dtype=torch.float16, device="cuda")
        if "C4" in hw:
            c4 = hw["C4"]
            unit[0] = "C4"
            self.c4 = dict(comp=put(c4["comp"]), offsets=put(c4["offsets"]), scales=put(c4["scales"]),
                           zeros=put(c4["zeros"]))
            self.c4_out = torch.empty(c4["rows"] * c4["cols"], dtype=torch.float16, device="cuda")
        if "C4u" in hw:
            c = hw["C4u"]
            unit[0] = "C4u"
            self.c4u = dict(packed=put(c["packed"]), scales=put(c["scales"]), zeros=put(c["zeros"]))
            self.c4u_out = torch.empty(c["rows"] * c["cols"], dtype=torch.float16, device="cuda")
        self.c5 = []
        if "C5" in hw:
            layer_elems = max(sum(m["rows"] * m["cols"] for m in mats) for mats in hw["C5"])
            self.c5_out = torch.empty(layer_elems, dtype=torch.float16, device="cuda")  # one reused layer buffer
            for li, mats in enumerate(hw["C5"]):
                unit[0] = ("C5", li)
                descs, base = [], 0
                for m in mats:
                    n = m["rows"] * m["cols"]
                    descs.append(dict(comp=put(m["comp"]), comp_bytes=int(m["comp"].size),
                                      block_offsets=put(m["offsets"]), scales=put(m["scales"]),
                                      zeros=put(m["zeros"]), out=self.c5_out[base:base + n], rows=m["rows"],
                                      cols=m["cols"], group_size=m["group_size"], block_bytes=m["block_bytes"]))
                    base += n
                self.c5.append(descs)
        # LZ4 workspace (sequence index), sized for the largest call: the
        # C5 index covers every layer (the layers are then expanded one by one)
        from weight_dequantization_b200 import lt_decode as L

        self.c5_first, tot = [], 0
        for descs in self.c5:
            self.c5_first.append(tot)
            tot += sum(L.desc_blocks(d) for d in descs)
        self.c5_blocks = tot
        self.c5_all = [d for descs in self.c5 for d in descs]
        nblk = [len(hw["C4"]["offsets"]) - 1] if "C4" in hw else []
        nblk += [sum(len(m["offsets"]) - 1 for m in mats) for mats in hw.get("C5", [])] + [tot]
        self.ws = torch.empty(max([L.lt_lz4_workspace_bytes(n) for n in nblk] + [16]), dtype=torch.uint8,
                              device="cuda")
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.status_host = torch.zeros(1, dtype=torch.int32).pin_memory() if pinned else None
        self.h2d_bytes = sum(int(p.numel() * p.element_size()) for p, _ in self.h2d)

    def units(self, two_step: bool = True):
        """The decode calls of one step, in order. two_step: C5 as one index
        call over all layers, then one expand call per layer; otherwise one
        decode call per layer."""
        hw = self.hw
        c5 = [("C5", i) for i in range(len(self.c5))]
        if two_step and c5:
            c5 = ["C5index"] + [("C5x", i) for i in range(len(self.c5))]
        return [u for u in STEP_CODECS if u in hw] + c5

    def run_unit(self, u, s):
        """Issue unit u's decode call on stream s."""
        from weight_dequantization_b200 import lt_decode as L

        hw = self.hw
        if u == "C1":
            c1 = hw["C1"]
            L.lt_dequant_int4(self.c1["packed"], self.c1["scales"], self.c1["zeros"], c1["rows"], c1["cols"],
                              c1["group_size"], self.c1_out, s)
        elif u == "C2":
            c2 = hw["C2"]
            L.lt_dequant_int8(self.c2["q"], self.c2["scales"], None, L.LT_SCALE_PER_ROW, c2["rows"], c2["cols"],
                              self.c2_out, s)
        elif u == "C3":
            c3 = hw["C3"]
            L.lt_zrle_decode(self.c3["enc"], int(c3["enc"].size), self.c3["offsets"], c3["n"], c3["chunk_elems"],
                             self.c3_out, self.status, s)
        elif u == "C4":
            c4 = hw["C4"]
            L.lt_lz4_int4_decode(self.c4["comp"], int(c4["comp"].size), self.c4["offsets"], c4["block_bytes"],
                                 self.c4["scales"], self.c4["zeros"], c4["rows"], c4["cols"], c4["group_size"],
                                 self.c4_out, self.ws, self.status, s)
        elif u == "C4u":
            c = hw["C4u"]
            L.lt_dequant_int4(self.c4u["packed"], self.c4u["scales"], self.c4u["zeros"], c["rows"], c["cols"],
                              c["group_size"], self.c4u_out, s)
        elif u == "C5index":
            L.lt_lz4_index_batch(self.c5_all, self.ws, s)
        elif u[0] == "C5x":
            L.lt_lz4_int4_expand_batch(self.c5[u[1]], self.ws, self.c5_blocks, self.c5_first[u[1]], self.status, s)
        else:
            L.lt_lz4_int4_decode_batch(self.c5[u[1]], self.ws, self.status, s)

    # one pass of the whole hot path; `ev` (optional) receives per-codec events
    def step(self, ev=None):
        torch = self.torch
        s = torch.cuda.current_stream()

        def mark(key):
            if ev is not None:
                e = torch.cuda.Event(enable_timing=True)
                e.record(s)
                ev.setdefault(key, []).append(e)

        mark("start")
        n = 0
        for u in self.units():
            self.run_unit(u, s)
            mark(u if u in STEP_CODECS else "C5")
            n += 1
        return n  # kernel launches of this step

    def e2e_step(self, cs, freed):
        """One step end to end: each unit's inputs are copied from pinned host
        memory on stream cs while the previous unit decodes on the current
        stream; a unit's copy waits until its buffers' last decode is done
        (`freed`: one event per unit, recorded after each decode)."""
        torch = self.torch
        s = torch.cuda.current_stream()
        for i, u in enumerate(self.units(two_step=False)):
            cs.wait_event(freed[i])
            with torch.cuda.stream(cs):
                for ph, d in self.unit_h2d.get(u, []):
                    d.copy_(ph, non_blocking=True)
            copied = torch.cuda.Event()
            copied.record(cs)
            s.wait_event(copied)
            self.run_unit(u, s)
            freed[i].record(s)
        self.download_status()

    def upload_inputs(self):
        for ph, d in self.h2d:
            d.copy_(ph, non_blocking=True)

    def download_status(self):
        self.status_host.copy_(self.status, non_blocking=True)


def launches_per_step(hw) -> int:
    # every call takes its vector path (no scalar tail launch): all element
    # counts are multiples of 8, groups multiples of 8, buffers 256-byte aligned
    n = 0
    for u in ("C1", "C4u"):
        if u in hw:
            c1 = hw[u]
            assert (c1["rows"] * c1["cols"]) % 8 == 0 and c1["group_size"] % 8 == 0
            n += 1
    if "C2" in hw:
        c2 = hw["C2"]
        assert (c2["rows"] * c2["cols"]) % 8 == 0 and c2["cols"] % 8 == 0
        n += 1
    # C3: one kernel; C4: parse + expand; C5: one index launch over all
    # layers, then one expand launch per layer
    n += ("C3" in hw) + 2 * ("C4" in hw) + ((1 + len(hw["C5"])) if hw.get("C5") else 0)
    return n


# ----------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ----------------------------------------------------------------------------

def oracle_sample_step(hw, frac: float):
    """Run the oracle on the first `frac` of every workload's units; returns
    (decoded bytes, seconds)."""
    import numpy as np

    import oracle

    t0 = time.perf_counter()
    dec = 0
    for u in ("C1", "C4u"):
        if u not in hw:
            continue
        c1 = hw[u]
        r1 = max(1, int(c1["rows"] * frac))
        n1 = r1 * c1["cols"]
        g1 = n1 // c1["group_size"]
        oracle.dequant_int4(c1["packed"][: n1 // 2], c1["scales"][:g1], c1["zeros"][:g1], r1, c1["cols"],
                            c1["group_size"])
        dec += 2 * n1
    if "C2" in hw:
        c2 = hw["C2"]
        r2 = max(1, int(c2["rows"] * frac))
        oracle.dequant_int8(c2["q"][: r2 * c2["cols"]], c2["scales"][:r2], None, True, r2, c2["cols"])
        dec += 2 * r2 * c2["cols"]
    if "C3" in hw:
        c3 = hw["C3"]
        nch = max(1, int((len(c3["offsets"]) - 1) * frac))
        n3 = min(c3["n"], nch * c3["chunk_elems"])
        oracle.zrle_decode(c3["enc"], c3["offsets"][: nch + 1], n3, c3["chunk_elems"])
        dec += 2 * n3

    def lz4_part(m):
        nb = max(1, int((len(m["offsets"]) - 1) * frac))
        s1 = int(m["offsets"][nb])
        codes = min(m["rows"] * m["cols"], nb * 2 * m["block_bytes"])
        g = codes // m["group_size"]
        oracle.lz4_int4_decode(m["comp"][:s1], m["offsets"][: nb + 1], m["block_bytes"], m["scales"][:g],
                               m["zeros"][:g], 1, codes, m["group_size"])
        return 2 * codes

    if "C4" in hw:
        dec += lz4_part(hw["C4"])
    for mats in hw.get("C5", []):
        for m in mats:
            dec += lz4_part(m)
    return dec, time.perf_counter() - t0


def oracle_sample_tasks(hw, frac: float, pieces: int):
    """The units of oracle_sample_step(hw, frac), cut into independent pieces
    (row, chunk and block ranges): a list of (callable, decoded bytes)."""
    import oracle

    tasks = []

    def split(n):
        k = max(1, min(pieces, n))
        return [(n * i // k, n * (i + 1) // k) for i in range(k) if n * i // k < n * (i + 1) // k]

    for u in ("C1", "C4u"):
        if u not in hw:
            continue
        c1 = hw[u]
        r1 = max(1, int(c1["rows"] * frac))
        cols, G = c1["cols"], c1["group_size"]
        for a, b in split(r1):
            tasks.append((lambda a=a, b=b, c1=c1, cols=cols, G=G: oracle.dequant_int4(
                c1["packed"][a * cols // 2:b * cols // 2], c1["scales"][a * cols // G:b * cols // G],
                c1["zeros"][a * cols // G:b * cols // G], b - a, cols, G), 2 * (b - a) * cols))
    if "C2" in hw:
        c2 = hw["C2"]
        r2 = max(1, int(c2["rows"] * frac))
        cols = c2["cols"]
        for a, b in split(r2):
            tasks.append((lambda a=a, b=b: oracle.dequant_int8(c2["q"][a * cols:b * cols], c2["scales"][a:b], None,
                                                                True, b - a, cols), 2 * (b - a) * cols))
    if "C3" in hw:
        c3 = hw["C3"]
        nch = max(1, int((len(c3["offsets"]) - 1) * frac))
        ce = c3["chunk_elems"]
        for a, b in split(nch):
            n_sub = min(c3["n"], b * ce) - a * ce
            tasks.append((lambda a=a, b=b, n_sub=n_sub: oracle.zrle_decode(c3["enc"], c3["offsets"][a:b + 1], n_sub,
                                                                            ce), 2 * n_sub))

    def lz4_tasks(m):
        nb = max(1, int((len(m["offsets"]) - 1) * frac))
        bb, G = m["block_bytes"], m["group_size"]
        for a, b in split(nb):
            c0 = 2 * a * bb
            codes = min(m["rows"] * m["cols"], 2 * b * bb) - c0
            g0, g1 = c0 // G, (c0 + codes + G - 1) // G
            tasks.append((lambda a=a, b=b, codes=codes, g0=g0, g1=g1: oracle.lz4_int4_decode(
                m["comp"], m["offsets"][a:b + 1], bb, m["scales"][g0:g1], m["zeros"][g0:g1], 1, codes, G),
                2 * codes))

    if "C4" in hw:
        lz4_tasks(hw["C4"])
    for mats in hw.get("C5", []):
        for m in mats:
            lz4_tasks(m)
    return tasks


# ----------------------------------------------------------------------------
# parity gate: one step's outputs against the oracle, every element
# ----------------------------------------------------------------------------

def _ulp_stats(got, want):
    """(elements, elements that differ, max binary16 ulp distance); +0 == -0
    and NaN == NaN as in the tests."""
    import numpy as np

    if got.shape != want.shape:
        return want.size, want.size, 1 << 20
    if np.array_equal(got, want):
        return want.size, 0, 0
    a, b = got.astype(np.int64), want.astype(np.int64)
    oa = np.where(a & 0x8000, -(a & 0x7FFF), a)
    ob = np.where(b & 0x8000, -(b & 0x7FFF), b)
    nan_a = ((a & 0x7C00) == 0x7C00) & ((a & 0x3FF) != 0)
    nan_b = ((b & 0x7C00) == 0x7C00) & ((b & 0x3FF) != 0)
    d = np.abs(oa - ob)
    d = np.where(nan_a & nan_b, 0, d)
    d = np.where(nan_a ^ nan_b, 1 << 20, d)
    return want.size, int((d > 0).sum()), int(d.max())


def _lz4_block_tasks(m, base_elem: int, per: int = 64):
    """(oracle call, first output element) per range of `per` blocks of
    matrix m, whose output starts at element base_elem of its buffer."""
    import numpy as np

    import oracle

    bb, G = m["block_bytes"], m["group_size"]
    n = m["rows"] * m["cols"]
    nb = len(m["offsets"]) - 1
    tasks = []
    for a in range(0, nb, per):
        b = min(nb, a + per)
        c0, c1 = 2 * a * bb, min(n, 2 * b * bb)
        s0, s1 = int(m["offsets"][a]), int(m["offsets"][b])
        offs = (m["offsets"][a:b + 1] - np.uint64(s0)).astype(np.uint64)
        g0, g1 = c0 // G, (c1 + G - 1) // G
        tasks.append((lambda m=m, s0=s0, s1=s1, offs=offs, g0=g0, g1=g1, c0=c0, c1=c1: oracle.lz4_int4_decode(
            m["comp"][s0:s1], offs, bb, m["scales"][g0:g1], m["zeros"][g0:g1], 1, c1 - c0, G), base_elem + c0))
    return tasks


def _row_tasks(fn, rows: int, cols: int, per_rows: int):
    return [(lambda a=a, b=min(rows, a + per_rows): fn(a, b), a * cols) for a in range(0, rows, per_rows)]


def parity_pass(dw, hw):
    """Issue one step's decode calls in order; after each call read its
    output back and compare every element with the oracle's (computed on
    all host cores, independent row / chunk / block ranges). Returns
    ({unit: outcome}, ok). Dequantized outputs must be within 1 binary16
    ulp of the oracle (0 expected), zero-run output bit for bit."""
    from concurrent.futures import ThreadPoolExecutor

    import numpy as np
    import torch

    import oracle

    s = torch.cuda.current_stream()
    threads = os.cpu_count() or 1
    outcome, ok = {}, True

    def host_bits(t):
        return t.cpu().view(torch.int16).numpy().view(np.uint16)

    def run(ex, tasks, got):
        n = bad = worst = 0
        for want_st, k0 in ex.map(lambda t: (t[0](), t[1]), tasks):
            want, st = want_st
            if st != 0:
                return None
            a, b, w = _ulp_stats(got[k0:k0 + want.size], want)
            n, bad, worst = n + a, bad + b, max(worst, w)
        return n, bad, worst

    def record(name, res, total, exact):
        nonlocal ok
        if res is None:
            outcome[name] = "oracle reported an error"
            ok = False
            return
        n, bad, worst = res
        good = n == total and worst <= (0 if exact else 1)
        ok = ok and good
        outcome[name] = (f"bit-exact, {n} of {total} elements" if bad == 0 and n == total else
                         f"{bad} of {n} elements differ (max {worst} ulp){'' if good else ': FAILED'}")

    with ThreadPoolExecutor(max_workers=threads) as ex:
        for u in dw.units():
            dw.run_unit(u, s)
            torch.cuda.synchronize()
            if u in ("C1", "C4u"):
                c = hw[u]
                cols, G = c["cols"], c["group_size"]
                fn = (lambda a, b, c=c, cols=cols, G=G: oracle.dequant_int4(
                    c["packed"][a * cols // 2:b * cols // 2], c["scales"][a * cols // G:b * cols // G],
                    c["zeros"][a * cols // G:b * cols // G], b - a, cols, G))
                out = dw.c1_out if u == "C1" else dw.c4u_out
                record(u, run(ex, _row_tasks(fn, c["rows"], cols, 64), host_bits(out)), c["rows"] * cols, False)
            elif u == "C2":
                c = hw["C2"]
                cols = c["cols"]
                fn = (lambda a, b: oracle.dequant_int8(c["q"][a * cols:b * cols], c["scales"][a:b], None, True,
                                                       b - a, cols))
                record(u, run(ex, _row_tasks(fn, c["rows"], cols, 128), host_bits(dw.c2_out)), c["rows"] * cols,
                       False)
            elif u == "C3":
                c = hw["C3"]
                ce, nch = c["chunk_elems"], len(c["offsets"]) - 1
                tasks = []
                for a in range(0, nch, 512):
                    b = min(nch, a + 512)
                    n_sub = min(c["n"], b * ce) - a * ce
                    tasks.append((lambda a=a, b=b, n_sub=n_sub: oracle.zrle_decode(c["enc"], c["offsets"][a:b + 1],
                                                                                    n_sub, ce), a * ce))
                record(u, run(ex, tasks, host_bits(dw.c3_out)), c["n"], True)
            elif u == "C4":
                c = hw["C4"]
                record(u, run(ex, _lz4_block_tasks(c, 0), host_bits(dw.c4_out)), c["rows"] * c["cols"], False)
            elif u == "C5index":
                continue
            else:  # one C5 layer, now in the reused buffer
                li = u[1]
                mats, base, tasks = hw["C5"][li], 0, []
                for m in mats:
                    tasks += _lz4_block_tasks(m, base)
                    base += m["rows"] * m["cols"]
                got = host_bits(dw.c5_out[:base])
                res = run(ex, tasks, got)
                prev = outcome.get("C5")
                if res is not None and isinstance(prev, tuple):
                    res = (prev[0] + res[0], prev[1] + res[1], max(prev[2], res[2]))
                outcome["C5"] = res if res is not None else None
                if li == len(hw["C5"]) - 1 or res is None:
                    total = sum(m["rows"] * m["cols"] for ms in hw["C5"] for m in ms)
                    record(f"C5 ({len(hw['C5'])} layers)", outcome.pop("C5"), total, False)
                    if res is None:
                        break
    torch.cuda.synchronize()
    st = int(dw.status.item())
    if st != 0:
        outcome["status"] = f"decoder status {st}"
        ok = False
    return outcome, ok


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline_threads(hw, frac: float):
    """The same oracle sample as cpu_baseline, spread over all host cores:
    independent pieces on a thread pool (the oracle's C code runs without
    the interpreter lock)."""
    from concurrent.futures import ThreadPoolExecutor

    threads = os.cpu_count() or 1
    tasks = oracle_sample_tasks(hw, frac, 4 * threads)
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        results = list(ex.map(lambda t: t[0](), tasks))
    dt = time.perf_counter() - t0
    if any(st != 0 for _, st in results):
        raise RuntimeError("the oracle reported an error in the threaded sample")
    dec = sum(b for _, b in tasks)
    return {"value": dec / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle", "cpu": cpu_model(),
            "sample": f"the cpu_baseline sample ({dec / 1e6:.1f} MB decoded) in {len(tasks)} independent pieces "
                      f"on {threads} threads, {dt:.2f} s"}


def cpu_baseline(hw, budget_s: float = 15.0):
    frac = 1.0 / 512
    dec, dt = oracle_sample_step(hw, frac)
    # scale the sample to the time budget (bounded)
    frac2 = min(0.25, frac * max(1.0, budget_s / max(dt, 1e-3)))
    if frac2 > frac * 1.5:
        frac = frac2
        dec, dt = oracle_sample_step(hw, frac)
    return {
        "value": dec / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle", "cpu": cpu_model(),
        "sample": f"first {frac:.4%} of the units (rows, chunks, 64 KB blocks) of every workload of one step "
                  f"({dec / 1e6:.1f} MB decoded in {dt:.1f} s, single-threaded plain C oracle)",
        "frac": frac,
    }


def cpu_baseline_value_dict():
    """The oracle on the whole value-dictionary workload, single-threaded."""
    import oracle
    from weight_dequantization_b200.synth import workloads as W

    d = W.v_value_dict()
    t0 = time.perf_counter()
    _, st = oracle.value_dict_decode(d["packed"], d["bits"], d["dictionary"], d["n"])
    dt = time.perf_counter() - t0
    if st != 0:
        raise RuntimeError("the oracle reported an error on the value-dictionary workload")
    return {"value": 2 * d["n"] / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle", "cpu": cpu_model(),
            "sample": f"the whole workload ({d['n']} elements, {2 * d['n'] / 1e6:.1f} MB decoded in {dt:.2f} s, "
                      f"single-threaded plain C oracle)"}


# ----------------------------------------------------------------------------
# arms
# ----------------------------------------------------------------------------

def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def workload_config(hw, layers, only=("C1", "C2", "C3", "C4", "C4u", "C5")):
    c5_codes = sum(m["rows"] * m["cols"] for mats in hw.get("C5", []) for m in mats)
    parts = {
        "C1": "C1 INT4 1M codes G256",
        "C2": "C2 INT8 8192x8192 per-row",
        "C3": "C3 zero-run 8x2048x11008",
        "C4": "C4 LZ4+INT4 4096x14336 G128",
        "C4u": "C4u INT4 4096x14336 G128 (C4's matrix uncompressed)",
        "C5": f"C5 {layers}-layer Llama-2-70B-shaped LZ4+INT4 G128 sweep (one reused layer buffer)",
    }
    return {
        "workload": "decode suite: " + " + ".join(parts[c] for c in parts if c in only) + " (64 KB LZ4 blocks)",
        "c5_codes": c5_codes,
        "l2": "inputs larger than L2 (each step touches ~16 GB; no flush)" if "C5" in only else
              "subset run: inputs may stay in L2 between steps",
    }


def c1_graph_steady_state(hw, peak: float, n_sets: int = 64, chains: int = 8, reps: int = 5):
    """C1 in steady state: one CUDA graph of `n_sets` C1 decodes, each on its
    own buffer set (together larger than L2), as `chains` independent chains
    of back-to-back decodes (so the small kernels overlap), replayed `reps`
    times after warm-up; device time per decode. A single C1 launch is
    bound by launch and ramp latency; this is the same kernel at
    throughput."""
    import numpy as np
    import torch

    from weight_dequantization_b200 import lt_decode as L

    c1 = hw["C1"]
    n = c1["rows"] * c1["cols"]

    def t(a):
        a = np.ascontiguousarray(a)
        return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()

    base = (t(c1["packed"]), t(c1["scales"]), t(c1["zeros"]))
    sets = [(base[0].clone(), base[1].clone(), base[2].clone(), torch.empty(n, dtype=torch.float16, device="cuda"))
            for _ in range(n_sets)]
    s = torch.cuda.Stream()
    side = [torch.cuda.Stream() for _ in range(chains)]

    def calls():
        fork = torch.cuda.Event()
        fork.record(s)
        joins = []
        for c, ss in enumerate(side):
            ss.wait_event(fork)
            for pk, sc, ze, out in sets[c::chains]:
                L.lt_dequant_int4(pk, sc, ze, c1["rows"], c1["cols"], c1["group_size"], out, ss)
            j = torch.cuda.Event()
            j.record(ss)
            joins.append(j)
        for j in joins:
            s.wait_event(j)

    with torch.cuda.stream(s):
        calls()  # eager warm-up (also fills the library's occupancy cache before capture)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        calls()
    for _, _, _, out in sets:  # poison the outputs: the replays must rewrite them
        out.view(torch.int16).fill_(0x7E00)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):  # a graph replays on the current stream
        for _ in range(3):
            g.replay()
        e0.record(s)
        for _ in range(reps):
            g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    per = e0.elapsed_time(e1) / 1e3 / (reps * n_sets)
    rd = nbytes(c1["packed"]) + nbytes(c1["scales"]) + nbytes(c1["zeros"])
    ref = torch.empty(n, dtype=torch.float16, device="cuda")
    with torch.cuda.stream(s):
        L.lt_dequant_int4(base[0], base[1], base[2], c1["rows"], c1["cols"], c1["group_size"], ref, s)
    torch.cuda.synchronize()
    same = all(torch.equal(o.view(torch.int16), ref.view(torch.int16)) for _, _, _, o in sets)
    del g
    return {"label": f"C1 steady state: CUDA graph of {n_sets} decodes on {n_sets} buffer sets "
                     f"({n_sets * (rd + 2 * n) / 1e6:.0f} MB, larger than L2) in {chains} independent chains of "
                     f"back-to-back decodes, {reps} replays",
            "us_per_call": per * 1e6, "decoded_GBps": 2 * n / per / 1e9,
            "hbm_frac_of_measured": (rd + 2 * n) / per / 1e9 / peak, "outputs_identical": bool(same)}


class L2Flush:
    """Before a timed call: write a 256 MB scratch buffer (twice L2), then
    read it back (a sum into a one-element tensor). The write evicts what
    the previous calls left in L2; the read evicts the write's dirty lines,
    so their write-back to HBM happens here and not inside the timed call,
    and L2 is left holding only clean lines of the scratch buffer."""

    def __init__(self, nbytes: int = 256 << 20):
        import torch
        self.buf = torch.empty(nbytes // 4, dtype=torch.int32, device="cuda")
        self.sink = torch.empty((), dtype=torch.int64, device="cuda")

    def __call__(self, r: int):
        import torch
        self.buf.fill_(r & 0xFF)
        torch.sum(self.buf, dim=0, dtype=torch.int64, out=self.sink)


def value_dict_timing(peak: float, reps: int = 30, warmup: int = 3):
    """The value-dictionary decode on its workload (4096 x 14336 4-bit
    indices with C4's code law, one 16-entry fp16 dictionary), timed per
    call with CUDA events on the launching stream; before every call a
    256 MB scratch write and read (not timed, L2Flush) flush L2."""
    import numpy as np
    import torch

    from weight_dequantization_b200 import lt_decode as L
    from weight_dequantization_b200.synth import workloads as W

    d = W.v_value_dict()
    n, bits = d["n"], d["bits"]
    packed = torch.from_numpy(d["packed"]).cuda()
    dictionary = torch.from_numpy(d["dictionary"].view(np.int16)).cuda()
    out = torch.empty(n, dtype=torch.float16, device="cuda")
    flush = L2Flush()
    s = torch.cuda.current_stream()
    times = []
    for r in range(warmup + reps):
        flush(r)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s)
        L.lt_value_dict_decode(packed, bits, dictionary, n, out, s)
        e1.record(s)
        torch.cuda.synchronize()
        if r >= warmup:
            times.append(e0.elapsed_time(e1) / 1e3)
    rd = int(d["packed"].nbytes + d["dictionary"].nbytes)
    wr = 2 * n
    med = statistics.median(times)
    del flush
    return {"label": f"value-dictionary decode: {d['rows']}x{d['cols']} {bits}-bit indices (C4's code law), "
                     f"one {1 << bits}-entry fp16 dictionary; L2 flushed before each of {reps} calls",
            "kernel": f"k_dict_vec<{bits}>", "us_per_call_median": med * 1e6, "us_per_call_min": min(times) * 1e6,
            "decoded_GBps": wr / med / 1e9, "bytes_read": rd, "bytes_written": wr,
            "hbm_frac_of_measured": (rd + wr) / med / 1e9 / peak,
            "hbm_frac_of_8TBps": (rd + wr) / med / 1e9 / NOMINAL_HBM_GBS}


def read_tflops_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured (cuBLAS bf16 burst; fp16 runs at the same tensor rate)"
    except Exception:
        return 1590.0, "fallback"


GEMM_SHAPES = (("q/o", 8192, 8192), ("k/v", 8192, 1024), ("gate/up", 8192, 28672), ("down", 28672, 8192))


def gemm_timing(hbm_peak: float, reps: int = 10, warmup: int = 3, shapes=GEMM_SHAPES, batch=(1, 16, 128, 4096)):
    """Fused INT4 decode -> GEMM (lt_int4_gemm) on the C5 weight shapes
    ([K, N] = [in, out], C4's code law, group 128) against decode-then-
    cuBLAS (lt_dequant_int4 into an fp16 buffer, then torch.matmul). Device
    time per call by CUDA events, median of `reps`, an L2 flush (L2Flush)
    before each call (not timed). Roofline: HBM bytes (x + packed
    codes + scales + zero points + out) against the measured copy peak, and
    2 M N K flops against the measured dense 16-bit tensor peak; the bound
    is whichever time is larger."""
    import numpy as np
    import torch

    from weight_dequantization_b200 import lt_decode as L
    from weight_dequantization_b200.synth import fp16_uniform, int4_gauss_groups_packed, u8_uniform

    tpeak, tkind = read_tflops_peak()
    s = torch.cuda.current_stream()
    flush = L2Flush()

    def timed(fn):
        ts = []
        for r in range(warmup + reps):
            flush(r)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(s)
            fn()
            e1.record(s)
            torch.cuda.synchronize()
            if r >= warmup:
                ts.append(e0.elapsed_time(e1) / 1e3)
        return statistics.median(ts)

    rows = []
    for name, K, N in shapes:
        G = 128
        packed = torch.from_numpy(int4_gauss_groups_packed(11, K * N)).cuda()
        scales = torch.from_numpy(fp16_uniform(11, K * N // G, 0.001, 0.1, stream=1).view(np.int16)).cuda()
        zeros = torch.from_numpy(u8_uniform(11, K * N // G, 0, 15, stream=2)).cuda()
        wbuf = torch.empty(K * N, dtype=torch.float16, device="cuda")
        for M in batch:
            x = torch.from_numpy(fp16_uniform(12, M * K, -1.0, 1.0, stream=7).view(np.int16)).cuda()
            x16 = x.view(torch.float16).view(M, K)
            out = torch.empty(M * N, dtype=torch.float16, device="cuda")
            wsb = L.lt_int4_gemm_workspace_bytes(M, N, K)
            ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")
            st = torch.zeros(1, dtype=torch.int32, device="cuda")
            t_fused = timed(lambda: L.lt_int4_gemm(x, M, K, packed, scales, zeros, N, G, out, ws, st, s))
            out_ref = torch.empty(M, N, dtype=torch.float16, device="cuda")

            def dec_then_mm():
                L.lt_dequant_int4(packed, scales, zeros, K, N, G, wbuf, s)
                torch.matmul(x16, wbuf.view(K, N), out=out_ref)

            t_base = timed(dec_then_mm)
            t_mm = timed(lambda: torch.matmul(x16, wbuf.view(K, N), out=out_ref))
            torch.cuda.synchronize()
            if int(st.item()) != 0:
                raise RuntimeError(f"lt_int4_gemm reported status {int(st.item())}")
            diff = (out.view(M, N).float() - out_ref.float()).abs()
            scale = out_ref.float().abs().max().item()
            byts = 2 * M * K + K * N // 2 + 3 * K * N // G + 2 * M * N
            flops = 2.0 * M * N * K
            t_hbm, t_tc = byts / (hbm_peak * 1e9), flops / (tpeak * 1e12)
            rows.append({"shape": name, "M": M, "K": K, "N": N, "us_fused": t_fused * 1e6,
                         "us_decode_then_cublas": t_base * 1e6, "us_cublas_alone": t_mm * 1e6,
                         "speedup_vs_decode_then_cublas": t_base / t_fused,
                         "TFLOPs_fused": flops / t_fused / 1e12, "GBps_fused": byts / t_fused / 1e9,
                         "bound": "tensor" if t_tc > t_hbm else "hbm",
                         "roofline_frac": max(t_hbm, t_tc) / t_fused, "splits_workspace_bytes": wsb,
                         "max_abs_diff_vs_cublas": diff.max().item(), "max_abs_out": scale})
            del x, out, out_ref, ws
        del packed, scales, zeros, wbuf
    del flush
    return {"label": "fused INT4 decode -> tcgen05 GEMM (lt_int4_gemm) vs lt_dequant_int4 + torch.matmul (cuBLAS) "
                     "on the C5 weight shapes; L2 flushed before each call; median of %d" % reps,
            "tensor_peak_TFLOPs": tpeak, "tensor_peak_kind": tkind, "hbm_peak_GBps": hbm_peak, "rows": rows}


def checksum_timing(dw, hw, peak: float, reps: int = 20, warmup: int = 3):
    """Per-block XXH3-64 on C4's compressed stream (448 blocks): the
    standalone verifier (lt_xxh3_blocks, one CTA per block) and the decode
    with the check fused in (lt_lz4_int4_decode_checked) against the plain
    fused decode. Device time by CUDA events, median of `reps`, an L2 flush
    (L2Flush) before each call (not timed)."""
    import numpy as np
    import torch

    from weight_dequantization_b200 import lt_decode as L

    c4 = hw["C4"]
    nb = len(c4["offsets"]) - 1
    secret = torch.from_numpy(np.random.default_rng(99).integers(0, 256, 192, dtype=np.uint8)).cuda()
    hashes = torch.zeros(nb, dtype=torch.int64, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    first = torch.full((1,), -1, dtype=torch.int64, device="cuda")
    s = torch.cuda.current_stream()
    comp_bytes = int(c4["comp"].size)
    L.lt_xxh3_blocks(dw.c4["comp"], comp_bytes, dw.c4["offsets"], nb, secret, 192, hashes, None, st, first, s)
    flush = L2Flush()

    def timed(fn):
        ts = []
        for r in range(warmup + reps):
            flush(r)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(s)
            fn()
            e1.record(s)
            torch.cuda.synchronize()
            if r >= warmup:
                ts.append(e0.elapsed_time(e1) / 1e3)
        return statistics.median(ts)

    def plain():
        L.lt_lz4_int4_decode(dw.c4["comp"], comp_bytes, dw.c4["offsets"], c4["block_bytes"], dw.c4["scales"],
                             dw.c4["zeros"], c4["rows"], c4["cols"], c4["group_size"], dw.c4_out, dw.ws, st, s)

    def checked():
        L.lt_lz4_int4_decode_checked(dw.c4["comp"], comp_bytes, dw.c4["offsets"], c4["block_bytes"],
                                     dw.c4["scales"], dw.c4["zeros"], c4["rows"], c4["cols"], c4["group_size"],
                                     dw.c4_out, secret, 192, hashes, dw.ws, st, first, s)

    t_hash = timed(lambda: L.lt_xxh3_blocks(dw.c4["comp"], comp_bytes, dw.c4["offsets"], nb, secret, 192, None,
                                            hashes, st, first, s))
    t_plain = timed(plain)
    t_checked = timed(checked)
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise RuntimeError(f"checksum leg: status {int(st.item())}")
    hb = comp_bytes + 8 * (nb + 1) + 8 * nb
    del flush
    return {"label": f"XXH3-64 per LZ4 block of C4 ({nb} blocks, {comp_bytes} compressed bytes, 192-byte secret); "
                     f"L2 flushed before each of {reps} calls",
            "kernel": "k_xxh3_blocks (one CTA per block)", "us_verify": t_hash * 1e6, "verify_GBps": hb / t_hash / 1e9,
            "verify_hbm_frac_of_measured": hb / t_hash / 1e9 / peak,
            "us_decode_plain": t_plain * 1e6, "us_decode_checked": t_checked * 1e6,
            "checked_overhead": t_checked / t_plain - 1.0}


def lz4_cliff_timing(dw, hw, reps: int = 10, warmup: int = 2):
    """Blocks with more LZ4 sequences than the index holds (512 per block),
    which the expanding CTA walks itself: 448 blocks of 64 KB (C4's count)
    of bytes uniform over 4 values, compressed by the generator's LZ4 into
    ~15,000 short sequences per block; raw decode (lt_lz4_decode) timed
    against the raw decode of C4's own compressed stream (~335 sequences per
    block). Device time by CUDA events, median of `reps`, L2 flushed before
    each call."""
    import numpy as np
    import torch

    from weight_dequantization_b200 import lt_decode as L
    from weight_dequantization_b200.synth import lz4_compress_blocks, u8_uniform

    nb = 448
    raw = u8_uniform(9, nb * 65536, 0, 3)
    comp, offs = lz4_compress_blocks(raw, 65536)
    dcomp = torch.from_numpy(comp).cuda()
    doffs = torch.from_numpy(offs.view(np.int64)).cuda()
    out = torch.empty(nb * 65536, dtype=torch.uint8, device="cuda")
    ws = torch.empty(L.lt_lz4_workspace_bytes(nb), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream()
    flush = L2Flush()
    c4 = hw["C4"]
    out4 = torch.empty(c4["packed_bytes"], dtype=torch.uint8, device="cuda")

    def timed(fn):
        ts = []
        for r in range(warmup + reps):
            flush(r)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(s)
            fn()
            e1.record(s)
            torch.cuda.synchronize()
            if r >= warmup:
                ts.append(e0.elapsed_time(e1) / 1e3)
        return statistics.median(ts)

    t_many = timed(lambda: L.lt_lz4_decode(dcomp, int(comp.size), doffs, 65536, out, nb * 65536, ws, st, s))
    t_c4 = timed(lambda: L.lt_lz4_decode(dw.c4["comp"], int(c4["comp"].size), dw.c4["offsets"], 65536, out4,
                                         c4["packed_bytes"], dw.ws, st, s))
    torch.cuda.synchronize()
    ok = int(st.item()) == 0 and bool(torch.equal(out, torch.from_numpy(raw).cuda()))
    del flush
    return {"label": f"LZ4 blocks beyond the 512-sequence index ({nb} x 64 KB of bytes uniform on 4 values, "
                     f"{comp.size} compressed bytes) against C4's stream, raw decode; L2 flushed before each call",
            "us_many_sequences": t_many * 1e6, "GBps_many_sequences": nb * 65536 / t_many / 1e9,
            "us_c4_raw": t_c4 * 1e6, "GBps_c4_raw": c4["packed_bytes"] / t_c4 / 1e9,
            "slowdown": t_many / t_c4, "output_matches_input": ok}


def stream_api_timing(hw, reps: int = 3):
    """The streaming API (LayerStreamer) over the C5 layers against
    sequential loading: streamed = each layer's host-to-device copy overlaps
    the previous layer's decode; sequential = each layer copied, then
    decoded, one after the other on one stream. Device time by CUDA events,
    median of `reps` runs each, inputs in pinned host memory."""
    import torch

    from weight_dequantization_b200.stream import LayerStreamer

    st = LayerStreamer(hw["C5"])
    s = torch.cuda.current_stream()

    def timed(fn):
        ts = []
        for r in range(reps + 1):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(s)
            fn()
            e1.record(s)
            torch.cuda.synchronize()
            if r:
                ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    t_stream = timed(lambda: st.run(stream=s))
    t_seq = timed(lambda: st.run_sequential(stream=s))
    status = st.status()
    h2d = sum(nb for _, nb, _ in st.layers)
    dec = sum(2 * m["rows"] * m["cols"] for mats in hw["C5"] for m in mats)
    res = {"label": f"LayerStreamer over {len(hw['C5'])} C5 layers from pinned host memory (two device slots, one "
                    f"reused output buffer) vs sequential copy-then-decode per layer; median of {reps} runs",
           "streamed_ms": t_stream, "sequential_ms": t_seq, "speedup": t_seq / t_stream,
           "h2d_bytes": h2d, "decoded_GBps_streamed": dec / t_stream / 1e6,
           "h2d_GBps_streamed": h2d / t_stream / 1e6, "status": status}
    del st
    return res


def run_lt(args, rank, world, local):
    import torch

    torch.cuda.set_device(local)
    dist = dist_init(world)
    from weight_dequantization_b200 import lt_decode as L

    L.load_library()
    only = tuple(x.strip() for x in args.only.split(",") if x.strip())
    hw = build_host_workload(rank, args.layers, only)
    (alg, layer_alg) = algorithmic_bytes(hw)
    dw = DeviceWorkload(hw, pinned=True)
    nlaunch = launches_per_step(hw)
    torch.cuda.synchronize()

    # warm-up
    for _ in range(max(args.warmup, 0)):
        dw.step()
    torch.cuda.synchronize()
    if int(dw.status.item()) != 0:
        raise RuntimeError(f"decode reported status {int(dw.status.item())} on the benchmark input")

    # parity gate: one more step, every output compared with the oracle; a
    # mismatch means no bench value
    if args.no_parity:
        parity, parity_ok = "not checked (--no-parity)", True
    else:
        t_par = time.perf_counter()
        parity, parity_ok = parity_pass(dw, hw)
        parity["seconds"] = round(time.perf_counter() - t_par, 1)
        parity["how"] = ("one step's calls in order, each output read back and compared element by element with "
                         "the oracle (all host cores); dequantized outputs within 1 binary16 ulp, zero-run bit for bit")
    if not parity_ok:
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": None, "unit": "GB/s", "n_gpus": world, "impl": "lt",
                              "parity": parity, "error": "parity failed: no bench value"}), flush=True)
        raise SystemExit(1)

    # timed region: K steps, device time by CUDA events on the launching stream
    clocks = ClockSampler(gpu_id_for(local))
    clocks.start()
    time.sleep(0.3)
    ev = {}
    s = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(s)
    for _ in range(args.steps):
        dw.step(ev)
    e1.record(s)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ck = clocks.stop()
    elapsed = e0.elapsed_time(e1) / 1e3
    elapsed = max_over_ranks(elapsed, dist)

    # per codec (device time of the launches, summed over steps): events are
    # recorded at the step start and after every launch, in launch order
    K = args.steps
    order = [c for c in STEP_CODECS if c in hw] + ["C5"] * ((1 + len(dw.c5)) if dw.c5 else 0)
    t_c = {c: 0.0 for c in alg}
    per_step = {c: [] for c in alg}  # device ms of the codec's launches in each step
    layer_t = []
    idx = {c: 0 for c in set(order)}
    for k in range(K):
        prev = ev["start"][k]
        step_c = {c: 0.0 for c in alg}
        for c in order:
            cur = ev[c][idx[c]]
            idx[c] += 1
            dt = prev.elapsed_time(cur)
            t_c[c] += dt
            step_c[c] += dt
            if c == "C5":
                layer_t.append(dt)
            prev = cur
        for c in alg:
            per_step[c].append(step_c[c])
    L5 = max(1, len(dw.c5))
    peak, peak_kind = read_peaks()
    per_codec = {}
    for c, (rd, wr) in alg.items():
        t = t_c[c] / 1e3 / K
        calls = L5 if c == "C5" else 1
        per_codec[c] = {"decoded_GBps": wr / t / 1e9, "us_per_call": t * 1e6 / calls,
                        "us_per_call_median": statistics.median(per_step[c]) * 1e3 / calls,
                        "us_per_call_min": min(per_step[c]) * 1e3 / calls,
                        "bytes_read": rd, "bytes_written": wr,
                        "hbm_frac_of_measured": (rd + wr) / t / 1e9 / peak,
                        "hbm_frac_of_8TBps": (rd + wr) / t / 1e9 / NOMINAL_HBM_GBS}
    decoded = sum(wr for _, wr in alg.values())
    total_decoded = sum_over_ranks(decoded * K, dist)
    value = total_decoded / elapsed / 1e9

    # roofline of the dominant kernel: the fused LZ4 decode, one launch per
    # C5 layer (the C4 launch when C5 is not run)
    if layer_t:
        avg_s = t_c["C5"] / 1e3 / K / L5  # a layer's expand launch + its share of the all-layer index launch
        launch_bytes = statistics.mean([rd + wr for rd, wr in layer_alg])
        kname = ("k_lz4_parse (one launch over all C5 layers) + k_lz4_expand (one launch per layer, 7 matrices): "
                 "per layer")
    elif "C4" in alg:
        avg_s = t_c["C4"] / 1e3 / K
        launch_bytes = sum(alg["C4"])
        kname = "k_lz4<fused> (C4)"
    else:
        c0 = next(iter(alg))
        avg_s = t_c[c0] / 1e3 / K
        launch_bytes = sum(alg[c0])
        kname = c0
    achieved = launch_bytes / avg_s / 1e9
    traffic = None
    if NCU_TRAFFIC["sources_sha256"] == kernel_sources_sha() and NCU_TRAFFIC["bytes_per_launch"] and layer_t:
        traffic = NCU_TRAFFIC["bytes_per_launch"]
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": traffic, "kernel": kname,
                "peak_kind": peak_kind, "algorithmic_bytes_per_launch": launch_bytes,
                "frac_of_8TBps": achieved / NOMINAL_HBM_GBS}

    # end-to-end: every step copies all its inputs from pinned host memory and
    # reads the status back; unit i + 1's copy overlaps unit i's decode
    torch.cuda.synchronize()
    dw.upload_inputs()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    KE = max(1, args.e2e_steps)
    cs = torch.cuda.Stream()
    f0.record(s)
    freed = []
    for _ in dw.units(two_step=False):  # every unit's buffers are free at the start of the timed region
        e = torch.cuda.Event()
        e.record(s)
        freed.append(e)
    for _ in range(KE):
        dw.e2e_step(cs, freed)
    f1.record(s)
    torch.cuda.synchronize()
    e2e_t = max_over_ranks(f0.elapsed_time(f1) / 1e3, dist)
    e2e_total = sum_over_ranks(decoded * KE, dist)
    e2e = {"value": e2e_total / e2e_t / 1e9, "unit": "GB/s", "h2d_bytes_per_step": dw.h2d_bytes,
           "d2h_bytes_per_step": 4, "steps": KE}
    if int(dw.status_host.item()) != 0:
        raise RuntimeError("decode reported an error in the end-to-end run")

    result = None
    if rank == 0:
        cpu = None
        cpu_thr = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline(hw)
            cpu_thr = cpu_baseline_threads(hw, cpu["frac"])
        c1g = c1_graph_steady_state(hw, peak) if "C1" in hw else None
        vd = value_dict_timing(peak) if "V" in only else None
        sapi = stream_api_timing(hw) if ("S" in only and hw.get("C5")) else None
        gshapes = tuple(x for x in GEMM_SHAPES if x[0] in args.gemm_shapes.split(","))
        gemm = gemm_timing(peak, shapes=gshapes, batch=tuple(int(m) for m in args.gemm_m.split(","))) \
            if "G" in only else None
        csum = checksum_timing(dw, hw, peak) if "C4" in hw else None
        cliff = lz4_cliff_timing(dw, hw) if "C4" in hw else None
        if vd is not None and world == 1 and not args.no_cpu_baseline:
            vd["cpu_baseline"] = cpu_baseline_value_dict()
        result = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": elapsed / K * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16", "data": "synthetic (seeded generators; value laws of the workloads)",
            "config": workload_config(hw, args.layers, only), "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": nlaunch * K, "clocks": {"sm_mhz": ck["sm_mhz"], "sm_max_mhz": ck["sm_max_mhz"],
                                                     "reasons": ck["reasons"], "samples": ck["samples"]},
            "per_codec": per_codec, "c1_graph": c1g, "value_dict": vd, "cpu_baseline_threads": cpu_thr,
            "parity": parity, "stream_api": sapi, "gemm": gemm, "checksum": csum, "lz4_many_sequences": cliff,
            "impl": "lt",
        }
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return result


def run_reference(args, rank, world):
    """The oracle (plain C, single thread) as the reference arm: each step is
    a bounded sample of the same workload, sized so the whole run stays
    within a few minutes."""
    if rank != 0:
        return None
    only = tuple(x.strip() for x in args.only.split(",") if x.strip())
    hw = build_host_workload(0, args.layers, only)
    steps = args.steps + args.warmup
    # calibrate: aim at ~90 s for all steps together
    dec, dt = oracle_sample_step(hw, 1.0 / 4096)
    per_step_budget = max(0.05, 90.0 / max(steps, 1))
    frac = min(0.25, (1.0 / 4096) * per_step_budget / max(dt, 1e-4))
    for _ in range(args.warmup):
        oracle_sample_step(hw, frac)
    tot_dec, tot_t = 0, 0.0
    for _ in range(args.steps):
        d, t = oracle_sample_step(hw, frac)
        tot_dec += d
        tot_t += t
    value = tot_dec / tot_t / 1e9
    sample = (f"first {frac:.5%} of the units of every workload per step, single-threaded plain C oracle "
              f"on the host ({tot_dec / max(args.steps, 1) / 1e6:.2f} MB decoded per step)")
    return {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": tot_t / max(args.steps, 1) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(hw, args.layers, only), "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    rank, world, local = dist_env()
    if args.impl == "reference":
        res = run_reference(args, rank, world)
    else:
        res = run_lt(args, rank, world, local)
    if res is not None and rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
