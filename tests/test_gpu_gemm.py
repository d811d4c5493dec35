"""GPU parity of the fused INT4 decode -> matrix multiply (lt_int4_gemm)
against the oracle's decode-then-multiply in double ("LoreToken-powered GPU
memory layer": decode + GEMM; "GPU Compression Pipeline - TDD Roadmap",
Phase 4.1: the decoded tensor used in input.matmul(weights)).

Tolerance: the kernel sums exact fp32 products on the tensor cores, whose
fp32 accumulation may truncate rather than round, so every addition is
taken to err by up to 2^-23 relative (u); over K terms in any order the sum
is then within gamma_K * sum|x w| of the exact one, gamma_K = K u / (1 - K u);
the one rounding to binary16 adds half an ulp of the result (2^-11 relative,
plus 2^-25 absolute for subnormal results)."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from tests._gpu import dev, host_bits, need_gpu, status_buf, torch
from weight_dequantization_b200 import lt_decode as L
from weight_dequantization_b200.synth import fp16_uniform, int4_gauss_groups_packed, u8_uniform

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    need_gpu()


def f16_to_f64(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def make_problem(M, K, N, G, seed, zeros=True):
    x = fp16_uniform(seed, M * K, -1.0, 1.0, stream=7)
    packed = int4_gauss_groups_packed(seed, K * N)
    scales = fp16_uniform(seed, K * N // G, 0.001, 0.1, stream=1)
    z = u8_uniform(seed, K * N // G, 0, 15, stream=2) if zeros else None
    return dict(M=M, K=K, N=N, G=G, x=x, packed=packed, scales=scales, zeros=z)


def run_gemm(p, split=True, dev_inputs=None):
    M, K, N, G = p["M"], p["K"], p["N"], p["G"]
    d = dev_inputs or dict(x=dev(p["x"]), packed=dev(p["packed"]), scales=dev(p["scales"]), zeros=dev(p["zeros"]))
    out = torch.full((M * N,), float("nan"), dtype=torch.float16, device="cuda")
    ws_bytes = L.lt_int4_gemm_workspace_bytes(M, N, K)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda") if (split and ws_bytes) else None
    st = status_buf()
    L.lt_int4_gemm(d["x"], M, K, d["packed"], d["scales"], d["zeros"], N, G, out, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return host_bits(out).reshape(M, N)


def sub_problem(p, rows, n0, n1):
    """The oracle's inputs for output rows `rows` and columns [n0, n1)."""
    K, N, G = p["K"], p["N"], p["G"]
    x = p["x"].reshape(p["M"], K)[rows]
    pk = p["packed"].reshape(K, N // 2)[:, n0 // 2:n1 // 2]
    sc = p["scales"].reshape(K, N // G)[:, n0 // G:n1 // G]
    z = None if p["zeros"] is None else p["zeros"].reshape(K, N // G)[:, n0 // G:n1 // G]
    return x, pk, sc, z


def check(got_bits, want, absum, K, what):
    u = 2.0 ** -23
    gamma = K * u / (1 - K * u)
    got = f16_to_f64(got_bits)
    bound = gamma * absum + 2.0 ** -11 * np.abs(want) + 2.0 ** -25
    err = np.abs(got - want)
    bad = ~(err <= bound)
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside the bound; worst excess "
                           f"{float(np.max(err - bound)):.3g} at {np.unravel_index(np.argmax(err - bound), err.shape)}")


@pytest.mark.parametrize("M,K,N,G,zeros", [(1, 64, 256, 32, True), (2, 1024, 512, 128, True), (3, 4096, 256, 64, False),
                                           (5, 128, 256, 128, True), (8, 2048, 768, 256, True), (9, 512, 256, 32, True),
                                           # small batches whose scale / zero-point rows are 16-byte multiples
                                           # (tiles of both by TMA), and a group of 96 (boxes straddling groups)
                                           (4, 512, 4096, 128, True), (6, 256, 512, 32, True), (2, 384, 768, 96, True),
                                           (7, 192, 2048, 64, False),
                                           # two blocks of 8 batch rows (9 .. 16 rows)
                                           (12, 512, 1024, 128, True), (16, 256, 4096, 128, True), (16, 320, 256, 32, False),
                                           (128, 256, 512, 64, False),
                                           (200, 512, 768, 256, True), (129, 1024, 256, 128, True),
                                           (300, 64, 1024, 32, False)])
def test_gemm_small_shapes_every_element(M, K, N, G, zeros):
    p = make_problem(M, K, N, G, seed=M * 7 + K, zeros=zeros)
    got = run_gemm(p)
    want, absum, st = oracle.int4_matmul(p["x"], M, p["packed"], p["scales"], p["zeros"], K, N, G)
    assert st == 0
    check(got, want, absum, K, f"M{M} K{K} N{N} G{G}")
    # without a workspace (no split of K) the result meets the same bound
    got1 = run_gemm(p, split=False)
    check(got1, want, absum, K, f"M{M} K{K} N{N} G{G} unsplit")


def test_gemm_identity_input_returns_the_decoded_weights():
    # x = the identity (K x K): out = W, and each output element is a single
    # exact product, so it equals lt_dequant_int4's output bit for bit
    K, N, G = 256, 512, 128
    p = make_problem(K, K, N, G, seed=3)
    eye = np.zeros((K, K), np.float16)
    np.fill_diagonal(eye, 1.0)
    p["x"] = eye.view(np.uint16).ravel()
    got = run_gemm(p)
    w = torch.empty(K * N, dtype=torch.float16, device="cuda")
    L.lt_dequant_int4(dev(p["packed"]), dev(p["scales"]), dev(p["zeros"]), K, N, G, w)
    torch.cuda.synchronize()
    assert np.array_equal(got.ravel(), host_bits(w))


@pytest.mark.parametrize("M,N", [(1, 512), (3, 512), (8, 512), (1, 4096), (5, 4096), (11, 512), (16, 4096)])
def test_gemm_small_batch_unit_rows_return_rows_of_the_decoded_weights(M, N):
    # batches of at most 16 rows take the mma.sync kernel: with x[m] the unit
    # vector e_(k_m), out[m] is row k_m of W, one exact product per element,
    # so it equals lt_dequant_int4's output bit for bit (N = 512: scales and
    # zero points copied word by word; N = 4096: by TMA)
    K, G = 1024, 128
    p = make_problem(M, K, N, G, seed=40 + M + N)
    ks = np.random.default_rng(M).choice(K, size=M, replace=False)
    x = np.zeros((M, K), np.float16)
    x[np.arange(M), ks] = 1.0
    p["x"] = x.view(np.uint16).ravel()
    got = run_gemm(p)
    w = torch.empty(K * N, dtype=torch.float16, device="cuda")
    L.lt_dequant_int4(dev(p["packed"]), dev(p["scales"]), dev(p["zeros"]), K, N, G, w)
    torch.cuda.synchronize()
    want = host_bits(w).reshape(K, N)[ks]
    assert np.array_equal(got, want)


C5_SHAPES = [("q", 8192, 8192), ("k", 8192, 1024), ("gate", 8192, 28672), ("down", 28672, 8192)]


@pytest.mark.parametrize("M", [1, 16, 128, 4096])
@pytest.mark.parametrize("name,K,N", C5_SHAPES)
def test_gemm_c5_shapes_sampled(name, K, N, M):
    # the Llama-2-70B-shaped weights of the C5 sweep ([in, out] = [K, N],
    # group 128), a batch of M rows; the oracle checks 3 rows x 256 columns
    # in each of 3 column blocks (first, a middle one, last)
    p = make_problem(M, K, N, 128, seed=K + N + M)
    got = run_gemm(p)
    rng = np.random.default_rng(M + N)
    rows = sorted(set([0, M - 1] + [int(r) for r in rng.integers(0, M, 1)]))
    blocks = sorted(set([0, N // 256 - 1, int(rng.integers(0, N // 256))]))
    for b in blocks:
        n0, n1 = 256 * b, 256 * b + 256
        x, pk, sc, z = sub_problem(p, rows, n0, n1)
        want, absum, st = oracle.int4_matmul(x.ravel(), len(rows), pk.ravel(), sc.ravel(),
                                             None if z is None else z.ravel(), K, 256, 128)
        assert st == 0
        check(got[rows][:, n0:n1], want, absum, K, f"{name} M{M} cols {n0}..{n1}")
