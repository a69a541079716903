"""Grouped (MoE) W8A8 GEMMs against the C++ oracle: many experts, each with its own weight and
scales, over one batch of token rows sorted by expert (ragged per-expert counts, experts without
tokens, counts that are not multiples of the 256-row tile).  Integer accumulators and slab
partials bit-exact; outputs within the criteria of tests/criteria.py."""
import numpy as np
import pytest
import torch

from oracle import ref_cpp as O
from activation_quantized_gemm_b200 import synth
from criteria import check_fp32, check_half
from gpu_util import dev, empty, host, setup_library

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    return setup_library()


def _problem(E, N, K, counts, seed):
    counts = np.asarray(counts, np.int64)
    M = int(counts.sum())
    x = synth.activation_bf16(max(M, 1), K, seed=seed, outlier_p=0.001, outlier_mult=50.0)[:M]
    w = np.stack([synth.weight_bf16(N, K, seed=seed + 1 + e) for e in range(E)])
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    return x, w, off


def _channel(q, x, w, off, ms=None, ns=None):
    E, N, K = w.shape
    M = x.shape[0]
    xq, sx = O.quant_act_token(x)
    wq = np.empty((E, N, K), np.int8)
    sw = np.empty((E, N), np.float32)
    for e in range(E):
        wq[e], sw[e] = O.quant_act_token(w[e])
    y = empty((M, N), torch.int16, 0x7FC0)
    acc = empty((M, N), torch.int32, 0x7FFFFFFF)
    offd = dev(off.astype(np.int32))
    q.i8q_gemm_w8a8_channel_grouped(dev(xq), dev(sx), dev(wq), dev(sw), offd, y, debug_acc=acc)
    y2 = empty((M, N), torch.int16, 0x7FC0)
    q.i8q_gemm_w8a8_channel_grouped(dev(xq), dev(sx), dev(wq), dev(sw), offd, y2)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    if ms is None:
        Y, A = O.gemm_w8a8_channel_grouped(xq, sx, wq, sw, off)
        assert np.array_equal(host(acc), A.astype(np.int32))
        check_half(host(y, np.uint16), Y, np.abs(Y), "bf16", f"grouped channel E={E} M={M}", strict=True)
    else:
        Y, A = O.gemm_w8a8_channel_grouped_at(xq, sx, wq, sw, off, ms, ns)
        assert np.array_equal(host(acc)[ms, ns], A.astype(np.int32))
        check_half(host(y, np.uint16)[ms, ns], Y, np.abs(Y), "bf16", f"grouped channel E={E} M={M}", strict=True)


def _block(q, x, w, off, ms=None, ns=None):
    E, N, K = w.shape
    M = x.shape[0]
    KB = K // 128
    xq, sx = O.quant_act_token_group(x)
    wq = np.empty((E, N, K), np.int8)
    sw = np.empty((E, (N + 127) // 128, KB), np.float32)
    for e in range(E):
        wq[e], sw[e] = O.quant_weight_block(w[e])
    ld = (M + 3) // 4 * 4
    sxd = np.zeros((KB, ld), np.float32)
    sxd[:, :M] = sx.T
    offd = dev(off.astype(np.int32))
    y32 = empty((M, N), torch.float32, float("nan"))
    yb = empty((M, N), torch.int16, 0x7FC0)
    dbg = empty((M, N, KB), torch.int32, 0x7FFFFFFF) if ms is None else None
    q.i8q_gemm_w8a8_block_grouped(dev(xq), dev(sxd), dev(wq), dev(sw), offd, y32, out=q.I8Q_OUT_FP32,
                                  debug_partials=dbg)
    q.i8q_gemm_w8a8_block_grouped(dev(xq), dev(sxd), dev(wq), dev(sw), offd, yb)
    torch.cuda.synchronize()
    if ms is None:
        Y, T, P = O.gemm_w8a8_block_grouped(xq, sx, wq, sw, off)
        assert np.array_equal(host(dbg), P.astype(np.int32))
        check_fp32(host(y32), Y, T, f"grouped block fp32 E={E} M={M}")
        check_half(host(yb, np.uint16), Y, T, "bf16", f"grouped block bf16 E={E} M={M}")
    else:
        Y, T, P = O.gemm_w8a8_block_grouped_at(xq, sx, wq, sw, off, ms, ns)
        check_fp32(host(y32)[ms, ns], Y, T, f"grouped block fp32 E={E} M={M}")
        check_half(host(yb, np.uint16)[ms, ns], Y, T, "bf16", f"grouped block bf16 E={E} M={M}")


CASES = [
    # (E, N, K, counts)
    (33, 264, 512, "dirichlet:1500"),       # many experts, ragged counts, some zero
    (8, 136, 384, [0, 300, 1, 0, 257, 0, 0, 3]),   # zero-token experts first and last, 256 +- 1
    (5, 7, 256, [40, 0, 0, 9, 1]),          # ragged N (unaligned output rows)
    (1, 520, 1024, [700]),                  # one expert = the dense GEMM
    (16, 256, 256, [0] * 15 + [20]),        # everything in the last expert
    (4, 128, 128, [1, 2, 3, 4]),            # decode-like: a few tokens per expert
]


def _counts(E, spec, seed):
    if isinstance(spec, str):
        total = int(spec.split(":")[1])
        c = synth.token_counts(E, total, seed=seed)
        if not (c == 0).any():
            c[seed % E] += c[(seed + 1) % E]
            c[(seed + 1) % E] = 0
        return c
    return np.asarray(spec, np.int64)


@pytest.mark.parametrize("case", range(len(CASES)))
def test_grouped_channel(q, case):
    E, N, K, spec = CASES[case]
    counts = _counts(E, spec, seed=case + 3)
    x, w, off = _problem(E, N, K, counts, seed=100 + case)
    _channel(q, x, w, off)


@pytest.mark.parametrize("case", range(len(CASES)))
def test_grouped_block(q, case):
    E, N, K, spec = CASES[case]
    counts = _counts(E, spec, seed=case + 3)
    x, w, off = _problem(E, N, K, counts, seed=200 + case)
    _block(q, x, w, off)


def test_grouped_matches_dense_entry_point(q):
    """With one expert the grouped call writes the same bits as the dense call."""
    M, N, K = 300, 264, 512
    x, w, off = _problem(1, N, K, [M], seed=300)
    xq, sx = O.quant_act_token(x)
    wq, sw = O.quant_act_token(w[0])
    y1 = empty((M, N), torch.int16)
    y2 = empty((M, N), torch.int16)
    q.i8q_gemm_w8a8_channel(dev(xq), dev(sx), dev(wq), dev(sw), y1)
    q.i8q_gemm_w8a8_channel_grouped(dev(xq), dev(sx), dev(wq[None]), dev(sw[None]), dev(off.astype(np.int32)), y2)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_grouped_offsets_out_of_range_stay_in_bounds(q):
    """Offsets past M (a caller's mistake) are clamped: nothing outside the [M, N] output is written."""
    E, N, K, M = 3, 136, 256, 50
    x, w, _ = _problem(E, N, K, [M], seed=400)
    xq, sx = O.quant_act_token(x)
    wq = np.stack([O.quant_act_token(w[e])[0] for e in range(E)])
    sw = np.stack([O.quant_act_token(w[e])[1] for e in range(E)])
    bad = np.array([0, 20, 10, 10_000], np.int32)          # decreasing, then far past M
    big = empty((M * N + 64,), torch.int16, 0x1234)
    q.i8q_gemm_w8a8_channel_grouped(dev(xq), dev(sx), dev(wq), dev(sw), dev(bad), big[: M * N].view(M, N))
    torch.cuda.synchronize()
    h = host(big).view(np.uint16)
    assert np.all(h[M * N:] == 0x1234)
    # rows 0..19 expert 0, rows 20..49 expert 2 (expert 1's range is empty after clamping)
    off = np.array([0, 20, 20, M])
    Y, A = O.gemm_w8a8_channel_grouped(xq, sx, wq, sw, off)
    check_half(h[: M * N].reshape(M, N), Y, np.abs(Y), "bf16", "clamped offsets", strict=True)


@pytest.mark.slow
def test_grouped_moe_down_proj_full_size(q):
    """DeepSeek-R1 MoE expert down-proj shape (N=7168, K=2048), 32 experts, 8192 routed token rows
    with ragged counts; outputs on sampled rows x columns."""
    E, N, K, total = 32, 7168, 2048, 8192
    counts = synth.token_counts(E, total, seed=7)
    x, w, off = _problem(E, N, K, counts, seed=500)
    rng = np.random.default_rng(8)
    ms = np.unique(np.concatenate([off[1:-1] - 1, off[1:-1], rng.integers(0, total, 200)]))
    ms = ms[(ms >= 0) & (ms < total)]
    ns = np.unique(np.concatenate([[0, 1, N - 1, 255, 256], rng.integers(0, N, 40)]))
    mm, nn = np.meshgrid(ms, ns, indexing="ij")
    _channel(q, x, w, off, mm.ravel(), nn.ravel())
    _block(q, x, w, off, mm.ravel(), nn.ravel())
