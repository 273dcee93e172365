"""GPU parity of the CUDA path (through the C-ABI) against the fp64 oracle.

Small shapes (several tiles, ragged tails) are compared element by element
against the full oracle.  The five named workloads run at full size in the
launch configuration the benchmark uses; the two smaller ones are compared in
full, the three large ones at oracle-exact sampled rows and ffn indices that
reach every output tile (parity_util.sample_indices).

Every workload runs in the default precision mode (the low half of the
activation pair in every product).  The fast mode (Y and dX from the high
half only) runs on the workloads where the header says it meets the bar.

Bar (elementwise, every output): max |gpu − oracle| ≤ 1e-2·(|oracle| + 1).
"""
import functools

import numpy as np
import pytest
import torch

from oracle import mlp_oracle as oracle
from tensor_transformer_mlp_bias_b200 import binding, block, inputs
from tests.parity_util import FFN_GROUP, ROW_GROUP, assert_close, bits, sample_indices, to_gpu

pytestmark = pytest.mark.gpu

ACCURATE, FAST = binding.ACCURATE, binding.FAST


def run_all(inp_gpu, t, mode=None):
    out = block.forward_backward(inp_gpu, t) if mode is None else block.forward_backward(inp_gpu, t, mode=mode)
    torch.cuda.synchronize()
    return out


def check_full(out, ref):
    for k in ("Y", "dX", "dA", "da", "dB", "db", "Z", "H"):
        assert_close(k, out[k], ref[k])
    assert_close("H + H_lo", out["H"].double() + out["H_lo"].double(), ref["H"])


# ------------------------------------------------------------------ small shapes, full oracle
SMALL = [
    # (T, h, f, t)  — ragged T, ragged N tiles (h or f not a multiple of 256), several K blocks
    (64, 256, 1024, 2),
    (1, 64, 128, 2),
    (200, 192, 384, 6),
    (333, 320, 1280, 5),
    (257, 512, 768, 3),
    (130, 128, 512, 8),
    # few weight-gradient tiles and a long token axis: their K loop is split into pieces
    (1024, 256, 1024, 2),
    (2048, 128, 512, 4),
]


@pytest.mark.parametrize("mode", [ACCURATE, FAST], ids=["accurate", "fast"])
@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "T%d_h%d_f%d_t%d" % s)
def test_small_shapes_full_oracle(shape, mode):
    T, h, f, t = shape
    inp = inputs.make_custom(T, h, f, seed=T + h + f + t)
    ref = oracle.full(inp)
    check_full(run_all(to_gpu(inp), t, mode), ref)


def test_tiny_workload_every_divisor():
    wl = inputs.WORKLOADS["tiny"]
    inp = inputs.make_inputs(wl)
    ref = oracle.full(inp)
    g = to_gpu(inp)
    for t in (1, 2, 4, 8, 16):
        check_full(run_all(g, t), ref)
        check_full(run_all(g, t, FAST), ref)


def test_empty_token_batch():
    T, h, f, t = 0, 128, 256, 2
    inp = to_gpu(inputs.make_custom(T, h, f))
    out = block.alloc_outputs(T, h, f)
    for k in ("dA", "dB", "da", "db"):
        out[k].fill_(7.0)
    ws = binding.make_workspace(T, h, f, t)
    block.forward(inp, t, out, ws)
    block.backward(inp, t, out, ws)
    binding.mlp_tp_check(ws)
    for k in ("dA", "dB", "da", "db"):
        assert bool((out[k] == 0).all()), k


# ------------------------------------------------------------------ named workloads
@functools.lru_cache(maxsize=1)
def _gpt2_medium():
    wl = inputs.WORKLOADS["gpt2-medium"]
    inp = inputs.make_inputs(wl)
    return inp, oracle.full(inp)


@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_gpt2_medium_full_oracle(t):
    inp, ref = _gpt2_medium()
    check_full(run_all(to_gpu(inp), t), ref)


def test_gpt2_medium_fast_mode():
    inp, ref = _gpt2_medium()
    check_full(run_all(to_gpu(inp), 8, FAST), ref)


@pytest.mark.parametrize("t", [16, 64])
def test_gpt2_medium_many_shards(t):
    """Up to 64 shards of 64 columns (the narrowest a shard may be): every shard's K segment is one K slice
    and each 256-column tile hands its accumulator to the epilogue t times."""
    inp, ref = _gpt2_medium()
    check_full(run_all(to_gpu(inp), t), ref)


@functools.lru_cache(maxsize=1)
def _sampled_reference(name):
    """Inputs, sampled indices and the oracle's exact values there; the ffn
    indices include both edges of every shard for each shard count the
    workload lists."""
    wl = inputs.WORKLOADS[name]
    inp = inputs.make_inputs(wl)
    rng = np.random.default_rng(1234)
    rows = sample_indices(wl.T, ROW_GROUP, rng)
    cols = np.unique(np.concatenate([sample_indices(wl.f, FFN_GROUP, rng, wl.f // t) for t in wl.shards]))
    return inp, rows, cols, oracle.sample_rows(inp, rows), oracle.sample_ffn(inp, cols)


def _sampled(name, t, mode=None):
    inp, rows, cols, sr, sc = _sampled_reference(name)
    out = run_all(to_gpu(inp), t, mode)
    r = torch.as_tensor(rows, device="cuda")
    c = torch.as_tensor(cols, device="cuda")
    assert_close("Y rows", out["Y"][r], sr["Y"])
    assert_close("Z rows", out["Z"][r], sr["Z"])
    assert_close("H rows", out["H"][r], sr["H"])
    assert_close("dX rows", out["dX"][r], sr["dX"])
    assert_close("dA cols", out["dA"][:, c], sc["dA"])
    assert_close("da cols", out["da"][c], sc["da"])
    assert_close("dB rows", out["dB"][c, :], sc["dB"])
    assert_close("db", out["db"], sc["db"])
    return out


@pytest.mark.parametrize("t", [1, 4, 8])
def test_h4096_sampled(t):
    _sampled("h4096", t)


@pytest.mark.parametrize("t", [1, 4, 8])
def test_h4096_fast_mode_sampled(t):
    """The bench's headline configuration: Y and dX from the high half."""
    _sampled("h4096", t, FAST)


def test_8p3b_class_sampled():
    # sqrt(f)·|B| is largest here: Y and dX need the low half of the pair, which the default mode uses
    _sampled("8.3b-class", 8)


def test_175b_class_sampled():
    _sampled("175b-class", 8)


def test_175b_class_fast_mode_sampled():
    _sampled("175b-class", 8, FAST)


# ------------------------------------------------------------------ invariants with no oracle
def test_t_independence_and_determinism():
    """Z, H, dA, dB, da, db do not depend on t bit for bit: shards are column
    or row blocks of the same GEMMs.  Y and dX differ across t only by the fp32
    shard-sum order.  A second run is bitwise identical."""
    T, h, f = 384, 512, 2048
    inp = to_gpu(inputs.make_custom(T, h, f, seed=5))
    outs = {t: run_all(inp, t) for t in (1, 2, 4, 8)}
    for t in (2, 4, 8):
        for k in ("Z", "H", "H_lo", "dA", "dB", "da", "db"):
            a, b = outs[t][k], outs[1][k]
            same = torch.equal(a, b) if a.dtype == torch.float32 else torch.equal(bits(a), bits(b))
            assert same, (k, t)
        for k in ("Y", "dX"):
            d = (outs[t][k].float() - outs[1][k].float()).abs()
            assert float(d.max()) <= 1e-2 * (1 + float(outs[1][k].float().abs().max())), (k, t)
    again = run_all(inp, 8)
    for k in again:
        a, b = again[k], outs[8][k]
        assert torch.equal(a, b) if a.dtype == torch.float32 else torch.equal(bits(a), bits(b)), k


@pytest.mark.parametrize("mode", [ACCURATE, FAST], ids=["accurate", "fast"])
def test_stage_entry_points_match_composite(mode):
    T, h, f, t = 300, 256, 1024, 4
    inp = to_gpu(inputs.make_custom(T, h, f, seed=9))
    comp = run_all(inp, t, mode)
    ws = binding.make_workspace(T, h, f, t)
    e = lambda *s: torch.empty(*s, dtype=torch.bfloat16, device="cuda")  # noqa: E731
    Z = torch.empty(T, f, dtype=torch.float32, device="cuda")
    H, H_lo, Y, dH, dH_lo = e(T, f), e(T, f), e(T, h), e(T, f), e(T, f)
    dX, dA, dB, da, db = e(T, h), e(h, f), e(f, h), e(f), e(h)
    binding.mlp_tp_fc1_forward(inp["X"], inp["A"], inp["a"], T, h, f, t, Z, H, H_lo, ws)
    binding.mlp_tp_fc2_forward(H, None if mode & FAST else H_lo, inp["B"], inp["b"], T, h, f, t, Y, ws)
    binding.mlp_tp_fc2_backward_data(inp["dY"], inp["B"], Z, T, h, f, t, dH, dH_lo, da, ws)
    binding.mlp_tp_fc2_backward_weight(H, H_lo, inp["dY"], T, h, f, t, dB, db, ws)
    binding.mlp_tp_fc1_backward_data(dH, None if mode & FAST else dH_lo, inp["A"], T, h, f, t, dX, ws)
    binding.mlp_tp_fc1_backward_weight(inp["X"], dH, dH_lo, T, h, f, t, dA, ws)
    binding.mlp_tp_check(ws)
    for k, v in dict(H=H, H_lo=H_lo, Y=Y, dX=dX, dA=dA, dB=dB, da=da, db=db).items():
        assert torch.equal(bits(v), bits(comp[k])), k
    assert torch.equal(Z, comp["Z"])
    # dH pair against the oracle's (dY·Bᵀ) ⊙ g'(Z)
    ref = oracle.f64(inp["dY"].cpu()) @ oracle.f64(inp["B"].cpu()).T
    Zr = oracle.f64(inp["X"].cpu()) @ oracle.f64(inp["A"].cpu()) + oracle.f64(inp["a"].cpu())
    assert_close("dH", dH.double() + dH_lo.double(), ref * oracle.gelu_grad(Zr))


def test_fc2_forward_without_bias():
    T, h, f, t = 128, 256, 512, 2
    inp = to_gpu(inputs.make_custom(T, h, f, seed=3))
    ws = binding.make_workspace(T, h, f, t)
    out = block.alloc_outputs(T, h, f)
    block.forward(inp, t, out, ws)
    Y0 = torch.empty_like(out["Y"])
    binding.mlp_tp_fc2_forward(out["H"], out["H_lo"], inp["B"], None, T, h, f, t, Y0, ws)
    binding.mlp_tp_check(ws)
    ref = oracle.forward(inp["X"].cpu(), inp["A"].cpu(), inp["a"].cpu(), inp["B"].cpu(), np.zeros(h))["Y"]
    assert_close("Y without b", Y0, ref)


def test_outputs_stay_inside_their_buffers():
    """Guard bands: every output lives inside a larger poisoned buffer; the
    bytes around it must be untouched after forward+backward."""
    T, h, f, t = 200, 192, 384, 3
    inp = to_gpu(inputs.make_custom(T, h, f, seed=4))
    shapes = {"Y": (T, h), "Z": (T, f), "H": (T, f), "H_lo": (T, f), "dX": (T, h), "dA": (h, f),
              "dB": (f, h), "da": (f,), "db": (h,)}
    pad = 4096  # elements of guard on each side, keeps 16-byte alignment
    poison = -12345.0
    bufs, out = {}, {}
    for k, s in shapes.items():
        n = int(np.prod(s))
        dt = torch.float32 if k == "Z" else torch.bfloat16
        buf = torch.full((n + 2 * pad,), poison, dtype=dt, device="cuda")
        bufs[k] = buf
        out[k] = buf[pad:pad + n].view(*s)
    block.forward_backward(inp, t, out)
    torch.cuda.synchronize()
    for k, buf in bufs.items():
        n = int(np.prod(shapes[k]))
        pv = torch.tensor(poison, dtype=buf.dtype)
        assert bool((buf[:pad].cpu() == pv).all()) and bool((buf[pad + n:].cpu() == pv).all()), k
    check_full(out, oracle.full(inputs.make_custom(T, h, f, seed=4)))


# ------------------------------------------------------------------ degenerate inputs
def test_zero_inputs_give_exact_zeros():
    """X = 0: Z = a, H = g(a) on every row, dA = Xᵀ·dH = 0 exactly.
    dY = 0: dX, dB, dH, da, db are exactly 0 and dA too."""
    T, h, f, t = 256, 256, 1024, 4
    host = inputs.make_custom(T, h, f, seed=41)
    host["X"].zero_()
    inp = to_gpu(host)
    out = run_all(inp, t)
    assert bool((out["dA"] == 0).all())
    ref = oracle.full(host)
    for k in ("Y", "Z", "H", "dX", "da", "dB", "db"):
        assert_close(k, out[k], ref[k])
    # every row of Z and H is the same (the bias and its GeLU)
    assert torch.equal(out["Z"], out["Z"][:1].expand_as(out["Z"]))
    host2 = inputs.make_custom(T, h, f, seed=42)
    host2["dY"].zero_()
    out2 = run_all(to_gpu(host2), t)
    for k in ("dX", "dA", "da", "dB", "db"):
        assert bool((out2[k] == 0).all()), k
    assert_close("Y", out2["Y"], oracle.forward(host2["X"], host2["A"], host2["a"], host2["B"], host2["b"])["Y"])


def test_large_preactivations_saturate_gelu():
    """|Z| up to ~40: GeLU passes positive values through and flushes negative
    ones to 0, g' goes to 1 and 0; no inf or NaN anywhere."""
    T, h, f, t = 128, 128, 512, 2
    host = inputs.make_custom(T, h, f, w_std=0.3, seed=43)
    host["X"] = (host["X"].float() * 3.0).to(torch.bfloat16)
    ref = oracle.full(host)
    assert float(np.abs(ref["Z"]).max()) > 20.0
    out = run_all(to_gpu(host), t)
    for k in out:
        assert bool(torch.isfinite(out[k].float()).all()), k
    check_full(out, ref)


# ------------------------------------------------------------------ seeded random shapes
def _random_shapes(n=12, seed=2024):
    """Ragged token counts, hidden sizes and shard widths (multiples of 64), 1-8 shards, both modes."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        t = int(rng.integers(1, 9))
        fs = 64 * int(rng.integers(1, 7))
        h = 64 * int(rng.integers(1, 11))
        T = int(rng.integers(1, 700))
        mode = ACCURATE if rng.random() < 0.5 else FAST
        out.append((T, h, fs * t, t, mode))
    return out


@pytest.mark.parametrize("shape", _random_shapes(), ids=lambda s: "T%d_h%d_f%d_t%d_m%d" % s)
def test_random_shapes_full_oracle(shape):
    T, h, f, t, mode = shape
    inp = inputs.make_custom(T, h, f, seed=T * 7 + h + f + t)
    check_full(run_all(to_gpu(inp), t, mode), oracle.full(inp))
