"""GPU: the streaming decode API (pinned host layers, two device staging
slots, one reused output buffer) against the oracle, layer by layer."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from tests._gpu import need_gpu, torch

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


def _f16_bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16).ravel()


def test_streamed_layers_decode_like_the_oracle():
    # the roadmap's streaming test, against the oracle (which sequential
    # decoding matches bit for bit): ten layers streamed through two staging
    # slots, each checked while it is in the reused buffer
    from weight_dequantization_b200.stream import LayerStreamer
    from weight_dequantization_b200.synth import workloads as W
    layers = W.c5_layers(layers=10, scale=1 / 256)  # the C5 shapes, 1/256 of the rows
    got = []
    st = LayerStreamer(layers)
    st.run(lambda i, views: got.append([v.clone() for v in views]))
    assert st.status() == 0
    for li, mats in enumerate(layers):
        for mi, m in enumerate(mats):
            want, s = oracle.lz4_int4_decode(m["comp"], m["offsets"], m["block_bytes"], m["scales"], m["zeros"],
                                             m["rows"], m["cols"], m["group_size"])
            assert s == 0
            assert np.array_equal(_f16_bits(got[li][mi]), want), (li, mi)
