"""bench.py's parity gate, run on the CPU: a stand-in for the device
workload whose "decodes" write the oracle's own output passes; the same with
one binary16 element off by 2 ulp, or one zero-run element changed by 1 ulp,
fails. No GPU: the device calls are replaced for the test."""
from __future__ import annotations

import numpy as np
import pytest

import bench
import oracle
from weight_dequantization_b200.synth import workloads as W

torch = pytest.importorskip("torch")


def _hw():
    c4 = W.c4_lz4_int4(scale=0.02, keep_packed=True)
    c4u = dict(kind="int4", rows=c4["rows"], cols=c4["cols"], group_size=c4["group_size"], packed=c4.pop("packed"),
               scales=c4["scales"], zeros=c4["zeros"])
    return {"C1": W.c1_int4(scale=0.25), "C2": W.c2_int8(scale=0.02), "C3": W.c3_zrle(scale=0.005), "C4": c4,
            "C4u": c4u, "C5": W.c5_layers(layers=2, scale=1 / 512)}


class FakeDeviceWorkload:
    """The parts of bench.DeviceWorkload the parity pass uses, with CPU
    tensors as outputs and the oracle as the 'decoder'."""

    def __init__(self, hw, plant=None):
        self.hw, self.plant = hw, plant
        f16 = lambda n: torch.zeros(n, dtype=torch.float16)  # noqa: E731
        self.c1_out = f16(hw["C1"]["rows"] * hw["C1"]["cols"])
        self.c2_out = f16(hw["C2"]["rows"] * hw["C2"]["cols"])
        self.c3_out = f16(hw["C3"]["n"])
        self.c4_out = f16(hw["C4"]["rows"] * hw["C4"]["cols"])
        self.c4u_out = f16(hw["C4u"]["rows"] * hw["C4u"]["cols"])
        self.c5_out = f16(max(sum(m["rows"] * m["cols"] for m in mats) for mats in hw["C5"]))
        self.status = torch.zeros(1, dtype=torch.int32)

    def units(self):
        return ["C1", "C2", "C3", "C4", "C4u", "C5index"] + [("C5x", i) for i in range(len(self.hw["C5"]))]

    @staticmethod
    def _put(t, bits):
        t[:bits.size].view(torch.int16).copy_(torch.from_numpy(bits.view(np.int16)))

    def run_unit(self, u, s):
        hw = self.hw
        if u in ("C1", "C4u"):
            c = hw[u]
            w, _ = oracle.dequant_int4(c["packed"], c["scales"], c["zeros"], c["rows"], c["cols"], c["group_size"])
            out = self.c1_out if u == "C1" else self.c4u_out
        elif u == "C2":
            c = hw["C2"]
            w, _ = oracle.dequant_int8(c["q"], c["scales"], None, True, c["rows"], c["cols"])
            out = self.c2_out
        elif u == "C3":
            c = hw["C3"]
            w, _ = oracle.zrle_decode(c["enc"], c["offsets"], c["n"], c["chunk_elems"])
            out = self.c3_out
        elif u == "C4":
            c = hw["C4"]
            w, _ = oracle.lz4_int4_decode(c["comp"], c["offsets"], c["block_bytes"], c["scales"], c["zeros"],
                                          c["rows"], c["cols"], c["group_size"])
            out = self.c4_out
        elif u == "C5index":
            return
        else:
            parts = []
            for m in hw["C5"][u[1]]:
                o, _ = oracle.lz4_int4_decode(m["comp"], m["offsets"], m["block_bytes"], m["scales"], m["zeros"],
                                              m["rows"], m["cols"], m["group_size"])
                parts.append(o)
            w, out = np.concatenate(parts), self.c5_out
        w = w.copy()
        if self.plant is not None and self.plant[0] == u:
            w[self.plant[1]] = (int(w[self.plant[1]]) + self.plant[2]) & 0xFFFF
        self._put(out, w)


@pytest.fixture
def no_cuda(monkeypatch):
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: None)


def test_parity_pass_accepts_the_oracles_own_output(no_cuda):
    hw = _hw()
    outcome, ok = bench.parity_pass(FakeDeviceWorkload(hw), hw)
    assert ok, outcome
    for u in ("C1", "C2", "C3", "C4", "C4u"):
        assert outcome[u].startswith("bit-exact"), outcome
    assert outcome["C5 (2 layers)"].startswith("bit-exact")


@pytest.mark.parametrize("plant,key", [((("C5x", 1), 777, 2), "C5 (2 layers)"), (("C3", 5000, 1), "C3"),
                                       (("C2", 123, 2), "C2")])
def test_parity_pass_refuses_a_planted_difference(no_cuda, plant, key):
    hw = _hw()
    if plant[0] == "C3":  # a non-zero element of the activations, so the change is 1 ulp of a literal
        plant = (plant[0], int(np.flatnonzero(hw["C3"]["x"])[0]), 1)
    outcome, ok = bench.parity_pass(FakeDeviceWorkload(hw, plant), hw)
    assert not ok
    assert "FAILED" in outcome[key], outcome
