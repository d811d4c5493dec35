"""GPU parity: LZ4 block decoding (raw bytes, bit-exact) and the fused
LZ4 -> INT4 -> fp16 decode (vs the oracle's decompress-then-dequantize)."""
from __future__ import annotations

import json
import os

import numpy as np
import pytest

import oracle
from tests._gpu import assert_f16_parity, dev, f16_out, host_bits, need_gpu, status_buf, torch
from tests._pins import hexbytes, liblz4, lz4_lib_compress
from weight_dequantization_b200 import lt_decode as L
from weight_dequantization_b200.synth import (fp16_uniform, int4_gauss_groups_packed, int4_uniform_packed,
                                              lz4_compress_block, lz4_compress_blocks, u8_uniform)
from weight_dequantization_b200.synth import workloads as W

pytestmark = pytest.mark.gpu
RNG = np.random.default_rng(13)


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


def workspace(n_blocks, mode="ws"):
    """The decoders' workspace: "ws" = enough for the sequence index,
    "none" = no workspace (every block walked by the expanding CTA)."""
    if mode == "none":
        return None
    return torch.empty(L.lt_lz4_workspace_bytes(n_blocks), dtype=torch.uint8, device="cuda")


def run_raw(comp, offsets, block_bytes, out_bytes, ws="ws"):
    out = torch.full((out_bytes + 16,), 0xEE, dtype=torch.uint8, device="cuda")
    stat = status_buf()
    L.lt_lz4_decode(dev(comp) if comp.size else None, int(comp.size), dev(offsets), block_bytes, out, out_bytes,
                    workspace(len(offsets) - 1, ws), stat)
    torch.cuda.synchronize()
    o = out.cpu().numpy()
    assert np.all(o[out_bytes:] == 0xEE), "write past the end of the output"
    return o[:out_bytes], int(stat.item())


def run_fused(d, zeros="use", out_offset=0, ws="ws"):
    z = d["zeros"] if zeros == "use" else None
    n = d["rows"] * d["cols"]
    out = f16_out(n, out_offset)
    stat = status_buf()
    L.lt_lz4_int4_decode(dev(d["comp"]), int(d["comp"].size), dev(d["offsets"]), d["block_bytes"], dev(d["scales"]),
                         dev(z), d["rows"], d["cols"], d["group_size"], out, workspace(len(d["offsets"]) - 1, ws),
                         stat)
    torch.cuda.synchronize()
    return host_bits(out), int(stat.item())


def oracle_fused(d, zeros="use"):
    z = d["zeros"] if zeros == "use" else None
    return oracle.lz4_int4_decode(d["comp"], d["offsets"], d["block_bytes"], d["scales"], z, d["rows"], d["cols"],
                                  d["group_size"])


def make_matrix(rows, cols, G, block_bytes, seed=1, law="gauss"):
    n = rows * cols
    packed = int4_gauss_groups_packed(seed, n) if law == "gauss" else int4_uniform_packed(seed, n)
    comp, offs = lz4_compress_blocks(packed, block_bytes)
    return dict(rows=rows, cols=cols, group_size=G, block_bytes=block_bytes, comp=comp, offsets=offs,
                packed=packed, scales=fp16_uniform(seed, n // G, 0.001, 0.1, stream=1),
                zeros=u8_uniform(seed, n // G, 0, 15, stream=2))


# --------------------------------------------------------------------------- raw LZ4

@pytest.mark.parametrize("ws", ["ws", "none"])
def test_lz4_handmade_blocks(golden_dir, ws):
    cases = json.load(open(os.path.join(golden_dir, "lz4_handmade.json")))["cases"]
    for c in cases:
        comp = np.frombuffer(hexbytes(c["comp"]), np.uint8)
        if "out" in c:
            want = hexbytes(c["out"])
        elif "out_repeat" in c:
            r = c["out_repeat"]
            want = hexbytes(r["unit"]) * r["count"] + hexbytes(r["extra"]) + hexbytes(r["tail"])
        else:
            want = None
        out_len = len(want) if want is not None else c["out_len"]
        offs = np.array([0, comp.size], np.uint64)
        bb = max(16, (out_len + 15) // 16 * 16)
        got, st = run_raw(comp, offs, bb, out_len, ws)
        _, st_o = oracle.lz4_block_decode(comp, out_len)
        assert st == st_o == c["status"], c["name"]
        if want is not None:
            assert got.tobytes() == want, c["name"]


@pytest.mark.parametrize("ws", ["ws", "none"])
def test_lz4_raw_c4_full_size_bit_exact(ws):
    d = W.c4_lz4_int4(keep_packed=True)
    got, st = run_raw(d["comp"], d["offsets"], d["block_bytes"], d["packed_bytes"], ws)
    assert st == 0
    assert np.array_equal(got, d["packed"])


@pytest.mark.parametrize("ws", ["ws", "none"])
@pytest.mark.parametrize("kind", ["0xab", "random_literals", "zeros", "max_offset"])
def test_lz4_roadmap_64k_blocks(kind, ws):
    if kind == "0xab":          # the roadmap's 64 KB block of 0xAB
        data = np.full(65536, 0xAB, np.uint8)
        comp = lz4_compress_block(data)
    elif kind == "random_literals":  # a block stored as literals only
        data = RNG.integers(0, 256, 65536, dtype=np.uint8)
        comp = lz4_compress_block(data, force_literals=True)
    elif kind == "zeros":
        data = np.zeros(65536, np.uint8)
        comp = lz4_compress_block(data)
    else:                        # the farthest match a 64 KB block can hold: offset 65500
        head = RNG.integers(0, 256, 65500, dtype=np.uint8)
        lit_ext = bytes([255] * ((65500 - 15) // 255)) + bytes([(65500 - 15) % 255])
        comp = np.frombuffer(bytes([0xFF]) + lit_ext + head.tobytes() + (65500).to_bytes(2, "little")
                             + bytes([31 - 4 - 15]) + bytes([0x50]) + b"tail!", np.uint8).copy()
        data = np.concatenate([head, head[:31], np.frombuffer(b"tail!", np.uint8)])
        assert data.size == 65536
        want, st_o = oracle.lz4_block_decode(comp, data.size)
        assert st_o == 0 and np.array_equal(want, data)
    got, st = run_raw(comp, np.array([0, comp.size], np.uint64), 65536, data.size, ws)
    assert st == 0 and np.array_equal(got, data)


@pytest.mark.skipif(liblz4() is None, reason="system liblz4 not present")
def test_lz4_decodes_blocks_from_the_system_lz4_library():
    blocks, raw = [], []
    for i in range(24):
        if i % 3 == 0:
            data = int4_gauss_groups_packed(i, 131072).tobytes()
        elif i % 3 == 1:
            data = RNG.integers(0, 4, 65536, dtype=np.uint8).tobytes()
        else:
            words = [b"lz4", b"block", b"decode", b"b200", b"nibble"]
            data = b"".join(words[j] for j in RNG.integers(0, 5, 20000))[:65536]
        blocks.append(lz4_lib_compress(data))
        raw.append(data)
    comp = np.frombuffer(b"".join(blocks), np.uint8)
    offs = np.concatenate([[0], np.cumsum([len(b) for b in blocks])]).astype(np.uint64)
    got, st = run_raw(comp, offs, 65536, 24 * 65536)
    assert st == 0
    assert got.tobytes() == b"".join(raw)


@pytest.mark.parametrize("n_bytes,block_bytes", [(1, 16), (100, 16), (5000, 4096), (200_001, 65536),
                                                 (300_000, 16384), (65536 * 3, 65536)])
def test_lz4_raw_ragged_sizes(n_bytes, block_bytes):
    data = int4_gauss_groups_packed(n_bytes, 2 * n_bytes)[:n_bytes]
    comp, offs = lz4_compress_blocks(data, block_bytes)
    got, st = run_raw(comp, offs, block_bytes, n_bytes)
    assert st == 0 and np.array_equal(got, data)


@pytest.mark.parametrize("ws", ["ws", "none"])
def test_lz4_corrupt_blocks_match_oracle_status(ws):
    data = int4_gauss_groups_packed(77, 131072)
    comp = lz4_compress_block(data)
    seen = set()
    for trial in range(80):
        c = comp.copy()
        if trial % 4 == 3:
            c = c[: int(RNG.integers(1, c.size))]
        else:
            for _ in range(1 + trial % 3):
                c[int(RNG.integers(0, c.size))] ^= np.uint8(1 << int(RNG.integers(0, 8)))
        want, st_o = oracle.lz4_block_decode(c, data.size)
        got, st_g = run_raw(c, np.array([0, c.size], np.uint64), 65536, data.size, ws)
        assert st_g == st_o, trial
        seen.add(st_o)
        if st_o == 0:
            assert np.array_equal(got, want)
    assert 4 in seen
    # offsets outside the stream
    got, st = run_raw(comp, np.array([0, comp.size + 10], np.uint64), 65536, data.size)
    assert st == L.LT_ERR_CORRUPT_STREAM
    got, st = run_raw(comp, np.array([10, 5], np.uint64), 65536, data.size)
    assert st == L.LT_ERR_CORRUPT_STREAM


# --------------------------------------------------------------------------- fused

@pytest.mark.parametrize("ws", ["ws", "none"])
def test_fused_c4_full_size(ws):
    d = W.c4_lz4_int4()
    want, st = oracle_fused(d)
    assert st == 0
    got, st_g = run_fused(d, ws=ws)
    assert st_g == 0
    assert_f16_parity(got, want, what="C4")


@pytest.mark.parametrize("rows,cols,G,block_bytes,law,zeros,out_offset", [
    (16, 8192, 128, 65536, "gauss", "use", 0),
    (16, 8192, 128, 65536, "gauss", None, 0),
    (8, 4096, 256, 16384, "uniform", "use", 0),
    (3, 4000, 8, 4096, "gauss", "use", 0),
    (5, 4002, 6, 4096, "gauss", "use", 0),        # groups not a multiple of 8: scalar epilogue
    (7, 4001, 4001, 16, "uniform", "use", 0),     # odd element count, tiny blocks
    (4, 4096, 128, 65536, "gauss", "use", 3),     # unaligned output
    (33, 2048, 64, 32768, "gauss", "use", 0),     # ragged last block
])
def test_fused_shapes(rows, cols, G, block_bytes, law, zeros, out_offset):
    d = make_matrix(rows, cols, G, block_bytes, seed=rows * cols, law=law)
    want, st = oracle_fused(d, zeros)
    assert st == 0
    got, st_g = run_fused(d, zeros, out_offset)
    assert st_g == 0
    assert_f16_parity(got, want, what=f"{rows}x{cols}/G{G}/B{block_bytes}")


def test_fused_corrupt_stream_reports_and_stays_in_bounds():
    d = make_matrix(64, 8192, 128, 65536, seed=3)
    assert len(d["offsets"]) == 5
    # block 1 cut short and block 2 starting inside block 1's bytes: both
    # decoders must fail (which error wins among several blocks is not fixed)
    offs = d["offsets"].copy()
    offs[2] = offs[1] + np.uint64(10)
    d["offsets"] = offs
    n = d["rows"] * d["cols"]
    buf = torch.full((n + 64,), 7.0, dtype=torch.float16, device="cuda")
    out = buf[:n]
    stat = status_buf()
    L.lt_lz4_int4_decode(dev(d["comp"]), int(d["comp"].size), dev(d["offsets"]), 65536, dev(d["scales"]),
                         dev(d["zeros"]), d["rows"], d["cols"], 128, out, workspace(4), stat)
    torch.cuda.synchronize()
    _, st_o = oracle_fused(d)
    assert st_o != 0
    assert int(stat.item()) in (L.LT_ERR_CORRUPT_STREAM, L.LT_ERR_SIZE_MISMATCH)
    assert torch.all(buf[n:] == 7.0)
    # blocks that are intact still decode exactly
    want, _ = oracle_fused(d)
    got = host_bits(out)
    assert np.array_equal(got[:131072], want[:131072])


@pytest.mark.parametrize("bad", [0, 5, 11])
def test_fused_one_bad_block_among_many_is_the_only_one_that_differs(bad):
    # one block of twelve replaced by random bytes of the same length: the
    # status is the oracle's (one bad block, so no race between errors), and
    # every other block's output is the oracle's, bit for bit -- the failure
    # stays inside the bad block's 131,072 elements
    d = make_matrix(192, 8192, 128, 65536, seed=91)
    nb = len(d["offsets"]) - 1
    assert nb == 12
    comp = d["comp"].copy()
    s0, s1 = int(d["offsets"][bad]), int(d["offsets"][bad + 1])
    comp[s0:s1] = np.random.default_rng(bad).integers(0, 256, s1 - s0, dtype=np.uint8)
    d["comp"] = comp
    want, st_o = oracle_fused(d)
    assert st_o != 0
    got, st_g = run_fused(d)
    assert st_g == st_o
    per = 131072  # elements per 64 KB block of INT4 codes
    keep = np.ones(d["rows"] * d["cols"], bool)
    keep[bad * per:(bad + 1) * per] = False
    assert np.array_equal(got[keep], want[keep])


def test_fused_batch_matches_per_matrix_oracle():
    # a Llama-shaped layer at 1/64 of the rows, one launch for all matrices
    mats = W.c5_layers(layers=1, scale=1 / 64)[0]
    outs, descs = [], []
    dev_refs = []
    for m in mats:
        n = m["rows"] * m["cols"]
        out = f16_out(n)
        refs = [dev(m["comp"]), dev(m["offsets"]), dev(m["scales"]), dev(m["zeros"])]
        dev_refs.append(refs)
        descs.append(dict(comp=refs[0], comp_bytes=int(m["comp"].size), block_offsets=refs[1], scales=refs[2],
                          zeros=refs[3], out=out, rows=m["rows"], cols=m["cols"], group_size=m["group_size"],
                          block_bytes=m["block_bytes"]))
        outs.append(out)
    stat = status_buf()
    nb = sum(len(m["offsets"]) - 1 for m in mats)
    L.lt_lz4_int4_decode_batch(descs, workspace(nb), stat)
    torch.cuda.synchronize()
    assert int(stat.item()) == 0
    for m, out in zip(mats, outs):
        want, st = oracle_fused(m)
        assert st == 0
        assert_f16_parity(host_bits(out), want, what=m["name"])


def test_fused_full_c5_layer_sampled_blocks():
    # one full-size layer in one launch (as the benchmark runs it); the oracle
    # checks a random sample of 64 KB blocks of every matrix one by one
    mats = W.c5_layers(layers=1)[0]
    total = sum(m["rows"] * m["cols"] for m in mats)
    buf = torch.empty(total, dtype=torch.float16, device="cuda")
    descs, keep, base = [], [], 0
    for m in mats:
        n = m["rows"] * m["cols"]
        refs = [dev(m["comp"]), dev(m["offsets"]), dev(m["scales"]), dev(m["zeros"])]
        keep.append(refs)
        descs.append(dict(comp=refs[0], comp_bytes=int(m["comp"].size), block_offsets=refs[1], scales=refs[2],
                          zeros=refs[3], out=buf[base:base + n], rows=m["rows"], cols=m["cols"],
                          group_size=m["group_size"], block_bytes=m["block_bytes"]))
        m["base"] = base
        base += n
    stat = status_buf()
    nb = sum(len(m["offsets"]) - 1 for m in mats)
    L.lt_lz4_int4_decode_batch(descs, workspace(nb), stat)
    torch.cuda.synchronize()
    assert int(stat.item()) == 0
    codes_per_block = 2 * 65536
    for m in mats:
        n_blocks = len(m["offsets"]) - 1
        for b in RNG.choice(n_blocks, size=min(12, n_blocks), replace=False):
            s0, s1 = int(m["offsets"][b]), int(m["offsets"][b + 1])
            g0 = b * codes_per_block // 128
            sub = dict(comp=m["comp"][s0:s1], offsets=np.array([0, s1 - s0], np.uint64), block_bytes=65536,
                       scales=m["scales"][g0:g0 + 1024], zeros=m["zeros"][g0:g0 + 1024], rows=1,
                       cols=codes_per_block, group_size=128)
            want, st = oracle_fused(sub)
            assert st == 0
            k0 = m["base"] + b * codes_per_block
            got = host_bits(buf[k0:k0 + codes_per_block])
            assert_f16_parity(got, want, what=f"{m['name']} block {b}")


@pytest.mark.parametrize("ws", ["ws", "none"])
@pytest.mark.parametrize("seed,n_blocks,block_bytes,last", [(1, 40, 65536, None), (2, 7, 65536, 12345),
                                                             (3, 30, 16384, 999), (4, 300, 4096, None)])
def test_lz4_random_sequence_blocks(seed, n_blocks, block_bytes, last, ws):
    # every match regime: offset 1, periodic 2..15, overlapping >= 16,
    # non-overlapping and far offsets; literal runs of every length class
    from tests._lz4gen import random_blocks
    comp, offs, raw = random_blocks(seed, n_blocks, block_bytes, last)
    got, st = run_raw(comp, offs, block_bytes, raw.size, ws)
    assert st == 0
    assert np.array_equal(got, raw)
    # and through the fused path: raw bytes are the packed codes
    n = 2 * raw.size
    G = 64 if n % 64 == 0 else 2
    d = dict(rows=1, cols=n, group_size=G, block_bytes=block_bytes, comp=comp, offsets=offs,
             scales=fp16_uniform(seed, n // G, -0.5, 0.5, stream=1), zeros=u8_uniform(seed, n // G, 0, 15, stream=2))
    want, st_o = oracle_fused(d)
    assert st_o == 0
    got, st_g = run_fused(d, ws=ws)
    assert st_g == 0
    assert_f16_parity(got, want, what="random blocks fused")


def test_lz4_blocks_with_more_sequences_than_the_index_holds():
    # short literals and short matches: thousands of sequences per 64 KB
    # block, beyond the workspace index; such blocks are walked by the CTA
    from tests._lz4gen import _sequence
    rng = np.random.default_rng(5)
    comps, raws = [], []
    for blk in range(6):
        out, comp = bytearray(), bytearray()
        while len(out) < 65536 - 40:
            lits = rng.integers(0, 256, int(rng.integers(1, 6)), dtype=np.uint8).tobytes()
            op = len(out) + len(lits)
            d = int(rng.integers(1, min(op, 2000) + 1))
            m = int(rng.integers(4, 12))
            comp += _sequence(lits, d, m)
            out += lits
            for _ in range(m):
                out.append(out[-d])
        tail = rng.integers(0, 256, 65536 - len(out), dtype=np.uint8).tobytes()
        comp += _sequence(tail, 0, 0)
        out += tail
        comps.append(bytes(comp))
        raws.append(bytes(out))
    comp = np.frombuffer(b"".join(comps), np.uint8).copy()
    offs = np.concatenate([[0], np.cumsum([len(c) for c in comps])]).astype(np.uint64)
    raw = np.frombuffer(b"".join(raws), np.uint8)
    want, st = oracle.lz4_decode_blocks(comp, offs, 65536, raw.size)
    assert st == 0 and np.array_equal(want, raw)
    got, st = run_raw(comp, offs, 65536, raw.size, "ws")
    assert st == 0 and np.array_equal(got, raw)


@pytest.mark.parametrize("shift", [1, 3, 8, 13])
def test_lz4_compressed_stream_not_16_byte_aligned(shift):
    from tests._lz4gen import random_blocks
    comp, offs, raw = random_blocks(9 + shift, 5, 65536, last=5000)
    dbuf = dev(np.concatenate([np.zeros(shift, np.uint8), comp]))
    out = torch.full((raw.size + 16,), 0xEE, dtype=torch.uint8, device="cuda")
    stat = status_buf()
    L.lt_lz4_decode(dbuf[shift:], int(comp.size), dev(offs), 65536, out, raw.size, workspace(len(offs) - 1), stat)
    torch.cuda.synchronize()
    assert int(stat.item()) == 0
    o = out.cpu().numpy()
    assert np.array_equal(o[:raw.size], raw) and np.all(o[raw.size:] == 0xEE)


# --------------------------------------------------------------------------- dependency depth

def _chain_block(n_matches: int, out_len: int, seed: int):
    """One LZ4 block whose matches form a single dependency chain: after 8
    literal bytes, every sequence is one literal byte and a 4-byte match of
    offset 5, which copies exactly the previous match's output; a literal
    run fills the block to `out_len` bytes (the format's end rules)."""
    from tests._lz4gen import _sequence

    rng = np.random.default_rng(seed)
    lits = rng.integers(0, 256, 8, dtype=np.uint8).tobytes()
    comp = bytearray()
    out = bytearray(lits)
    first = True
    for _ in range(n_matches):
        lit = rng.integers(0, 256, 1, dtype=np.uint8).tobytes()
        seq_lits = (lits + lit) if first else lit
        first = False
        out += lit
        for _ in range(4):
            out.append(out[-5])
        comp += _sequence(seq_lits, 5, 4)
    tail = rng.integers(0, 256, out_len - len(out), dtype=np.uint8).tobytes()
    assert len(tail) >= 12
    comp += _sequence(tail, 0, 0)
    out += tail
    return np.frombuffer(bytes(comp), np.uint8).copy(), np.frombuffer(bytes(out), np.uint8).copy()


@pytest.mark.parametrize("ws", ["ws", "none"])
@pytest.mark.parametrize("n_matches", [100, 400])
def test_lz4_long_match_dependency_chains(n_matches, ws):
    # 100 chained matches: 100 match levels, copied level by level (CTA-wide,
    # then the last ones by one warp); 400: the levels saturate and the block
    # is replayed in stream order. Both must give the oracle's bytes.
    comp, want = _chain_block(n_matches, 2048, seed=n_matches)
    got_o, st_o = oracle.lz4_block_decode(comp, want.size)
    assert st_o == 0 and np.array_equal(got_o, want)
    got, st = run_raw(comp, np.array([0, comp.size], np.uint64), 2048, want.size, ws)
    assert st == 0 and np.array_equal(got, want)
    # the same block through the fused decode: 2 x 2048 codes, G 128
    d = dict(rows=2, cols=2048, group_size=128, block_bytes=2048, comp=comp, offsets=np.array([0, comp.size], np.uint64),
             scales=fp16_uniform(n_matches, 32, 0.001, 0.1, stream=1), zeros=u8_uniform(n_matches, 32, 0, 15, stream=2))
    got_f, st_f = run_fused(d, ws=ws)
    want_f, st_of = oracle_fused(d)
    assert st_f == st_of == 0
    assert_f16_parity(got_f, want_f, what="fused decode of a dependency chain")


# --------------------------------------------------------------------------- two-step decode

def test_index_then_expand_in_slices_matches_oracle():
    # one index call over three matrices, then the matrices decoded in two
    # slices of that index (as the C5 sweep does with its layers)
    mats = [make_matrix(64, 8192, 128, 65536, seed=71), make_matrix(48, 4096, 128, 65536, seed=72),
            make_matrix(32, 8192, 128, 32768, seed=73)]
    descs, outs = [], []
    for m in mats:
        out = f16_out(m["rows"] * m["cols"], 0)
        outs.append(out)
        descs.append(dict(comp=dev(m["comp"]), comp_bytes=int(m["comp"].size), block_offsets=dev(m["offsets"]),
                          scales=dev(m["scales"]), zeros=dev(m["zeros"]), out=out, rows=m["rows"], cols=m["cols"],
                          group_size=m["group_size"], block_bytes=m["block_bytes"]))
    blocks = [L.desc_blocks(d) for d in descs]
    total = sum(blocks)
    index = torch.empty(L.lt_lz4_workspace_bytes(total), dtype=torch.uint8, device="cuda")
    L.lt_lz4_index_batch(descs, index)
    stat = status_buf()
    L.lt_lz4_int4_expand_batch(descs[:1], index, total, 0, stat)
    L.lt_lz4_int4_expand_batch(descs[1:2], index, total, blocks[0], stat)
    # the last slice has only 32 KB blocks, so its window is smaller than the
    # one the index was built for: its blocks are walked by the expanding CTA
    L.lt_lz4_int4_expand_batch(descs[2:], index, total, blocks[0] + blocks[1], stat)
    torch.cuda.synchronize()
    assert int(stat.item()) == 0
    for m, out in zip(mats, outs):
        want, st = oracle_fused(m)
        assert st == 0
        assert_f16_parity(host_bits(out), want, what="index + expand")
    # a stream error the index finds is reported by the expand covering its block
    bad = dict(mats[2])
    comp = bad["comp"].copy()
    comp[int(bad["offsets"][1]):int(bad["offsets"][2])] = 0xFF  # block 1: every token claims a long literal run
    bad["comp"] = comp
    descs[2] = dict(descs[2], comp=dev(comp))
    L.lt_lz4_index_batch(descs, index)
    stat0, stat1 = status_buf(), status_buf()
    L.lt_lz4_int4_expand_batch(descs[:2], index, total, 0, stat0)
    L.lt_lz4_int4_expand_batch(descs[2:], index, total, blocks[0] + blocks[1], stat1)
    torch.cuda.synchronize()
    _, st_o = oracle_fused(bad)
    assert int(stat0.item()) == 0
    assert int(stat1.item()) == st_o != 0


# --------------------------------------------------------------------------- both parse paths

@pytest.mark.parametrize("n_blocks", [40, 700])
def test_lz4_parse_paths_agree_with_the_oracle_and_report_the_same_errors(n_blocks):
    # A launch with few blocks per SM walks each block staged whole in shared
    # memory; one with many blocks per SM (more than 4 per SM here) streams
    # each block through a small ring. Both must decode every regime exactly
    # and report a damaged block with the oracle's status.
    from tests._lz4gen import random_blocks
    comp, offs, raw = random_blocks(60 + n_blocks, n_blocks, 4096)
    got, st = run_raw(comp, offs, 4096, raw.size, "ws")
    assert st == 0 and np.array_equal(got, raw)
    for blk, pos in ((n_blocks - 3, 0), (n_blocks // 2, 17)):
        bad = comp.copy()
        s0, s1 = int(offs[blk]), int(offs[blk + 1])
        bad[s0 + pos:s1] = 0xFF  # every token claims a long literal run past the block
        want, st_o = oracle.lz4_decode_blocks(bad, offs, 4096, raw.size)
        got, st_g = run_raw(bad, offs, 4096, raw.size, "ws")
        assert st_o != 0 and st_g == st_o
        keep = np.ones(raw.size, bool)
        keep[blk * 4096:(blk + 1) * 4096] = False
        assert np.array_equal(got[keep], raw[keep])
