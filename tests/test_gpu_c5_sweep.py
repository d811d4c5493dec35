"""GPU parity of the full-size 8-layer Llama-2-70B-shaped sweep, run exactly
as the benchmark runs it: one lt_lz4_index_batch over the blocks of all 8
layers (52,224 blocks), then one lt_lz4_int4_expand_batch per layer into one
reused fp16 buffer ("GPU Compression Pipeline - TDD Roadmap", Phase 2.1,
large tensors; the sweep of the Llama-2-70B-shaped configuration).

Two whole layers are compared with the oracle element by element, and 64
random 64 KB blocks of every other layer, each read back while that layer
is in the reused buffer."""
from __future__ import annotations

import numpy as np
import pytest

from tests._gpu import assert_f16_parity, dev, host_bits, need_gpu, status_buf, torch
from tests._oracle_threads import lz4_int4_block_range, pieces, pool
from weight_dequantization_b200 import lt_decode as L
from weight_dequantization_b200.synth import workloads as W

pytestmark = pytest.mark.gpu

FULL_LAYERS = (0, 5)
SAMPLED_BLOCKS = 64


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


def test_c5_sweep_index_once_expand_per_layer_matches_oracle():
    layers = W.c5_layers()  # 8 full-size layers, the benchmark's seed
    assert len(layers) == 8
    layer_elems = max(sum(m["rows"] * m["cols"] for m in mats) for mats in layers)
    buf = torch.empty(layer_elems, dtype=torch.float16, device="cuda")
    keep, descs_by_layer = [], []
    for mats in layers:
        descs, base = [], 0
        for m in mats:
            n = m["rows"] * m["cols"]
            refs = [dev(m["comp"]), dev(m["offsets"]), dev(m["scales"]), dev(m["zeros"])]
            keep.append(refs)
            descs.append(dict(comp=refs[0], comp_bytes=int(m["comp"].size), block_offsets=refs[1], scales=refs[2],
                              zeros=refs[3], out=buf[base:base + n], rows=m["rows"], cols=m["cols"],
                              group_size=m["group_size"], block_bytes=m["block_bytes"]))
            m["base"] = base
            base += n
        descs_by_layer.append(descs)
    first, total = [], 0
    for descs in descs_by_layer:
        first.append(total)
        total += sum(L.desc_blocks(d) for d in descs)
    assert total == 8 * 6528
    index = torch.empty(L.lt_lz4_workspace_bytes(total), dtype=torch.uint8, device="cuda")
    L.lt_lz4_index_batch([d for descs in descs_by_layer for d in descs], index)
    rng = np.random.default_rng(2024)
    host = torch.empty(layer_elems, dtype=torch.float16).pin_memory()
    with pool() as ex:
        for li, mats in enumerate(layers):
            stat = status_buf()
            buf.fill_(float("nan"))  # every element must be rewritten by this layer's expand
            L.lt_lz4_int4_expand_batch(descs_by_layer[li], index, total, first[li], stat)
            host.copy_(buf, non_blocking=True)
            torch.cuda.synchronize()
            assert int(stat.item()) == 0, f"layer {li}: status {int(stat.item())}"
            got = host.view(torch.int16).numpy().view(np.uint16)
            # (matrix, first block, last block) ranges to compare
            if li in FULL_LAYERS:
                ranges = [(m, a, b) for m in mats for a, b in pieces(len(m["offsets"]) - 1, 64)]
            else:
                nb = [len(m["offsets"]) - 1 for m in mats]
                picks = rng.choice(sum(nb), size=SAMPLED_BLOCKS, replace=False)
                cum = np.cumsum([0] + nb)
                ranges = []
                for p in sorted(int(x) for x in picks):
                    mi = int(np.searchsorted(cum, p, side="right")) - 1
                    ranges.append((mats[mi], p - int(cum[mi]), p - int(cum[mi]) + 1))
            results = list(ex.map(lambda r: (r, lz4_int4_block_range(*r)), ranges))
            checked = 0
            for (m, a, b), (want, st) in results:
                assert st == 0
                k0 = m["base"] + 2 * a * m["block_bytes"]
                assert_f16_parity(got[k0:k0 + want.size], want, what=f"layer {li} {m['name']} blocks {a}..{b}")
                checked += want.size
            if li in FULL_LAYERS:
                assert checked == sum(m["rows"] * m["cols"] for m in mats)
