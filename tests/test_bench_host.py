"""Host-side pieces of bench.py that run without a GPU: the threaded oracle
baseline covers exactly the units of the single-threaded sample, and
decoding them in pieces gives the same output as one call."""
from __future__ import annotations

import numpy as np

import bench
import oracle
from weight_dequantization_b200.synth import workloads as W


def _small_workloads():
    return {"C1": W.c1_int4(scale=0.25), "C2": W.c2_int8(scale=0.02), "C3": W.c3_zrle(scale=0.01),
            "C4": W.c4_lz4_int4(scale=0.1)}


def test_threaded_oracle_sample_covers_the_same_units():
    hw = _small_workloads()
    frac = 0.3
    dec, _ = bench.oracle_sample_step(hw, frac)
    tasks = bench.oracle_sample_tasks(hw, frac, 5)
    assert sum(b for _, b in tasks) == dec
    assert all(st == 0 for (_, st) in (t() for t, _ in tasks))


def test_lz4_pieces_decode_like_one_call():
    m = W.c4_lz4_int4(scale=0.1)
    frac = 0.5
    nb = max(1, int((len(m["offsets"]) - 1) * frac))
    s1 = int(m["offsets"][nb])
    codes = min(m["rows"] * m["cols"], nb * 2 * m["block_bytes"])
    g = codes // m["group_size"]
    whole, st = oracle.lz4_int4_decode(m["comp"][:s1], m["offsets"][: nb + 1], m["block_bytes"], m["scales"][:g],
                                       m["zeros"][:g], 1, codes, m["group_size"])
    assert st == 0
    pieces = [t() for t, _ in bench.oracle_sample_tasks({"C4": m}, frac, 3)]
    assert np.array_equal(np.concatenate([o for o, _ in pieces]), whole)


def test_zero_run_pieces_decode_like_one_call():
    c3 = W.c3_zrle(scale=0.01)
    frac = 1.0
    nch = len(c3["offsets"]) - 1
    whole, st = oracle.zrle_decode(c3["enc"], c3["offsets"], c3["n"], c3["chunk_elems"])
    assert st == 0 and nch > 3
    pieces = [t() for t, _ in bench.oracle_sample_tasks({"C3": c3}, frac, 4)]
    assert np.array_equal(np.concatenate([o for o, _ in pieces]), whole)


def test_value_dictionary_oracle_baseline_covers_the_workload():
    r = bench.cpu_baseline_value_dict()
    assert r["kind"] == "oracle" and r["cores"] == 1 and r["value"] > 0
    assert str(W.v_value_dict()["n"]) in r["sample"]
