"""GPU parity of the fp16 + e4m3 mode (MLP_TP_FP8) against the fp64 oracle.

The mode keeps H and dH as fp16 plus an e4m3 residual and runs the weight
gradients as an fp16 product plus an 8-bit (kind::f8f6f4) residual product
into one accumulator; Y and dX take one fp16 product each.  Same bar as every
other mode, max |gpu − oracle| ≤ 1e-2·(|oracle| + 1), on small and ragged
shapes (full oracle: ragged token counts exercise the 128-token e4m3 stages'
tails), on all five named workloads (the two small ones in full, the three
large ones at sampled rows and ffn indices that reach every output tile),
and on the degenerate inputs.  Exact invariants check the scale machinery:
scaling dY by a power of two scales every gradient by the same power, bit
for bit, and the stage calls reproduce the composite call bit for bit.
"""
import numpy as np
import pytest
import torch

from oracle import mlp_oracle as oracle
from tensor_transformer_mlp_bias_b200 import binding, block, inputs
from tests.parity_util import assert_close, bits, to_gpu, worst_ratio
from tests.test_parity import SMALL, _gpt2_medium, _sampled_reference

pytestmark = pytest.mark.gpu

FP8 = binding.FP8


def run_fp8(inp_gpu, t):
    out = block.forward_backward(inp_gpu, t, mode=FP8)
    torch.cuda.synchronize()
    return out


def h_value(out):
    """H as the mode keeps it: fp16 plus the e4m3 residual / 2^7."""
    return out["H"].double() + out["H_lo"].float().double() / 128.0


def check_full(out, ref):
    for k in ("Y", "dX", "dA", "da", "dB", "db", "Z", "H"):
        assert_close(k, out[k], ref[k])
    assert_close("H16 + H8/2^7", h_value(out), ref["H"])


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "T%d_h%d_f%d_t%d" % s)
def test_small_shapes_full_oracle(shape):
    T, h, f, t = shape
    inp = inputs.make_custom(T, h, f, seed=T + h + f + t)
    check_full(run_fp8(to_gpu(inp), t), oracle.full(inp))


@pytest.mark.parametrize("shape", [(127, 256, 512, 2), (129, 192, 768, 3), (385, 64, 256, 1), (640, 320, 640, 5)],
                         ids=lambda s: "T%d_h%d_f%d_t%d" % s)
def test_token_tails_of_the_8bit_stages(shape):
    """Token counts just below and above a multiple of the 128-token e4m3
    stage: the last stage is partly out of range and reads zeros."""
    T, h, f, t = shape
    inp = inputs.make_custom(T, h, f, seed=3 * T + h)
    check_full(run_fp8(to_gpu(inp), t), oracle.full(inp))


def test_tiny_workload_every_divisor():
    wl = inputs.WORKLOADS["tiny"]
    inp = inputs.make_inputs(wl)
    ref = oracle.full(inp)
    g = to_gpu(inp)
    for t in (1, 2, 4, 8, 16):
        check_full(run_fp8(g, t), ref)


@pytest.mark.parametrize("t", [1, 8, 64])
def test_gpt2_medium_full_oracle(t):
    """t = 64: shards of 64 columns, the narrowest allowed (one K slice per shard segment of Y and dX)."""
    inp, ref = _gpt2_medium()
    check_full(run_fp8(to_gpu(inp), t), ref)


def _sampled(name, t):
    inp, rows, cols, sr, sc = _sampled_reference(name)
    out = run_fp8(to_gpu(inp), t)
    r = torch.as_tensor(rows, device="cuda")
    c = torch.as_tensor(cols, device="cuda")
    assert_close("Y rows", out["Y"][r], sr["Y"])
    assert_close("Z rows", out["Z"][r], sr["Z"])
    assert_close("H rows", h_value(out)[r], sr["H"])
    assert_close("dX rows", out["dX"][r], sr["dX"])
    assert_close("dA cols", out["dA"][:, c], sc["dA"])
    assert_close("da cols", out["da"][c], sc["da"])
    assert_close("dB rows", out["dB"][c, :], sc["dB"])
    assert_close("db", out["db"], sc["db"])


@pytest.mark.parametrize("t", [1, 8])
def test_h4096_sampled(t):
    _sampled("h4096", t)


def test_8p3b_class_sampled():
    """Where the fast mode exceeds the bar: the fp16 products of Y and dX keep
    11 bits, which is enough."""
    _sampled("8.3b-class", 8)


def test_175b_class_sampled():
    _sampled("175b-class", 8)


def test_empty_token_batch():
    T, h, f, t = 0, 128, 256, 2
    inp = to_gpu(inputs.make_custom(T, h, f))
    out = block.alloc_outputs(T, h, f, mode=FP8)
    for k in ("dA", "dB", "da", "db"):
        out[k].fill_(7.0)
    ws = binding.make_workspace_mode(T, h, f, t, FP8)
    block.forward(inp, t, out, ws, FP8)
    block.backward(inp, t, out, ws, FP8)
    binding.mlp_tp_check(ws)
    for k in ("dA", "dB", "da", "db"):
        assert bool((out[k] == 0).all()), k


def test_stage_entry_points_match_composite():
    T, h, f, t = 300, 256, 1024, 4
    inp = to_gpu(inputs.make_custom(T, h, f, seed=9))
    comp = run_fp8(inp, t)
    ws = binding.make_workspace_mode(T, h, f, t, FP8)
    e = lambda *s: torch.empty(*s, dtype=torch.bfloat16, device="cuda")  # noqa: E731
    Z = torch.empty(T, f, dtype=torch.float32, device="cuda")
    H, dH = (torch.empty(T, f, dtype=torch.float16, device="cuda") for _ in range(2))
    H_lo, dH_lo = (torch.empty(T, f, dtype=torch.uint8, device="cuda") for _ in range(2))
    Y, dX, dA, dB, da, db = e(T, h), e(T, h), e(h, f), e(f, h), e(f), e(h)
    binding.mlp_tp_fp8_prepare_forward(inp["B"], T, h, f, t, ws)
    binding.mlp_tp_fc1_forward_fp8(inp["X"], inp["A"], inp["a"], T, h, f, t, Z, H, H_lo, ws)
    binding.mlp_tp_fc2_forward_fp8(H, inp["b"], T, h, f, t, Y, ws)
    binding.mlp_tp_fp8_prepare_backward(inp["dY"], inp["X"], inp["A"], inp["B"], T, h, f, t, ws)
    binding.mlp_tp_fc2_backward_data_fp8(inp["dY"], inp["B"], Z, T, h, f, t, dH, dH_lo, da, ws)
    binding.mlp_tp_fc2_backward_weight_fp8(H, H_lo, inp["dY"], T, h, f, t, dB, db, ws)
    binding.mlp_tp_fc1_backward_data_fp8(dH, T, h, f, t, dX, ws)
    binding.mlp_tp_fc1_backward_weight_fp8(dH, dH_lo, T, h, f, t, dA, ws)
    binding.mlp_tp_check(ws)
    for k, v in dict(Y=Y, dX=dX, dA=dA, dB=dB, da=da, db=db).items():
        assert torch.equal(bits(v), bits(comp[k])), k
    assert torch.equal(Z, comp["Z"]) and torch.equal(bits(H), bits(comp["H"]))
    assert torch.equal(H_lo, comp["H_lo"].view(torch.uint8))
    # dH16 + dH8/2^7 is dH·sH: against the oracle's (dY·Bᵀ) ⊙ g'(Z), up to the one power-of-two scale
    ref = oracle.f64(inp["dY"].cpu()) @ oracle.f64(inp["B"].cpu()).T
    Zr = oracle.f64(inp["X"].cpu()) @ oracle.f64(inp["A"].cpu()) + oracle.f64(inp["a"].cpu())
    dh_ref = ref * oracle.gelu_grad(Zr)
    got = dH.double() + dH_lo.view(torch.float8_e4m3fn).float().double() / 128.0
    s = float(np.exp2(np.round(np.log2(float(got.abs().max()) / np.abs(dh_ref).max()))))
    assert s >= 1.0 and s == 2.0 ** round(np.log2(s))
    assert_close("dH·sH / sH", got / s, dh_ref)


def test_recompute_matches_saved_activations():
    T, h, f, t = 320, 256, 768, 3
    inp = to_gpu(inputs.make_custom(T, h, f, seed=17))
    saved = run_fp8(inp, t)
    ws = binding.make_workspace_mode(T, h, f, t, FP8, recompute=True)
    e = lambda *s: torch.empty(*s, dtype=torch.bfloat16, device="cuda")  # noqa: E731
    Y, dX, dA, dB, da, db = e(T, h), e(T, h), e(h, f), e(f, h), e(f), e(h)
    binding.mlp_tp_forward_recompute(inp["X"], inp["A"], inp["a"], inp["B"], inp["b"], T, h, f, t, FP8, Y, ws)
    binding.mlp_tp_backward_recompute(inp["dY"], inp["X"], inp["A"], inp["a"], inp["B"], T, h, f, t, FP8,
                                      dX, dA, da, dB, db, ws)
    binding.mlp_tp_check(ws)
    for k, v in dict(Y=Y, dX=dX, dA=dA, dB=dB, da=da, db=db).items():
        assert torch.equal(bits(v), bits(saved[k])), k


def test_gradient_scale_invariance():
    """dY·2^-20 (tiny gradients, far below fp16's normal range) gives every
    gradient ·2^-20 bit for bit: sY and sH grow by 2^20, so the fp16 and e4m3
    copies, and every product, are the same bits."""
    T, h, f, t = 384, 256, 1024, 4
    host = inputs.make_custom(T, h, f, seed=21)
    small = dict(host)
    small["dY"] = (host["dY"].float() * 2.0 ** -20).to(torch.bfloat16)
    a = run_fp8(to_gpu(host), t)
    b = run_fp8(to_gpu(small), t)
    for k in ("Y", "Z"):
        assert torch.equal(a[k], b[k]), k
    for k in ("dX", "dA", "dB", "da", "db"):
        assert torch.equal(a[k].float() * 2.0 ** -20, b[k].float()), k


def test_zero_inputs_give_exact_zeros():
    T, h, f, t = 256, 256, 1024, 4
    host = inputs.make_custom(T, h, f, seed=41)
    host["X"].zero_()
    out = run_fp8(to_gpu(host), t)
    assert bool((out["dA"] == 0).all())
    ref = oracle.full(host)
    for k in ("Y", "Z", "dX", "da", "dB", "db"):
        assert_close(k, out[k], ref[k])
    host2 = inputs.make_custom(T, h, f, seed=42)
    host2["dY"].zero_()
    out2 = run_fp8(to_gpu(host2), t)
    for k in ("dX", "dA", "da", "dB", "db"):
        assert bool((out2[k] == 0).all()), k


def test_large_preactivations():
    """|Z| up to ~40 (GeLU saturated) with weights ~N(0, 0.3): inside the
    mode's range.  The weight gradients (fp16 + e4m3 residual, about 15 bits)
    and Z, H meet the bar; Y and dX, one fp16 product each (11 bits of H and
    dH), exceed it on entries near 0 here.  That is the mode's documented
    limit (the accurate mode keeps 16 bits there); the bound below records it."""
    T, h, f, t = 128, 128, 512, 2
    host = inputs.make_custom(T, h, f, w_std=0.3, seed=43)
    host["X"] = (host["X"].float() * 3.0).to(torch.bfloat16)
    ref = oracle.full(host)
    assert float(np.abs(ref["Z"]).max()) > 20.0
    out = run_fp8(to_gpu(host), t)
    for k in ("dA", "da", "dB", "db", "Z", "H"):
        assert_close(k, out[k], ref[k])
    assert_close("H16 + H8/2^7", h_value(out), ref["H"])
    for k in ("Y", "dX"):
        w = worst_ratio(out[k], ref[k])
        assert 0.0 < w < 4.0, (k, w)


def test_activation_beyond_the_range_is_reported():
    """|H| >= 2^13: the e4m3 residual would saturate; mlp_tp_check reports
    MLP_ERR_RANGE (the values stay finite, nothing faults)."""
    T, h, f, t = 128, 128, 512, 2
    host = inputs.make_custom(T, h, f, w_std=1.0, seed=44)
    host["X"] = (host["X"].float() * 1000.0).to(torch.bfloat16)
    inp = to_gpu(host)
    out = block.alloc_outputs(T, h, f, mode=FP8)
    ws = binding.make_workspace_mode(T, h, f, t, FP8)
    block.forward(inp, t, out, ws, FP8)
    with pytest.raises(binding.MlpError) as err:
        binding.mlp_tp_check(ws)
    assert err.value.status == 9 and "range" in str(err.value)
    binding.mlp_tp_check(ws)  # the status word was cleared


def test_binding_refuses_bf16_activations_in_fp8_calls():
    T, h, f, t = 64, 256, 1024, 2
    inp = to_gpu(inputs.make_custom(T, h, f, seed=1))
    ws = binding.make_workspace_mode(T, h, f, t, FP8)
    Hb = torch.empty(T, f, dtype=torch.bfloat16, device="cuda")
    Y = torch.empty(T, h, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        binding.mlp_tp_fc2_forward_fp8(Hb, inp["b"], T, h, f, t, Y, ws)


def _random_shapes(n=10, seed=2025):
    """Ragged token counts (not multiples of the 128-token e4m3 stage), hidden sizes and shard widths."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n):
        t = int(rng.integers(1, 9))
        fs = 64 * int(rng.integers(1, 7))
        h = 64 * int(rng.integers(1, 11))
        T = int(rng.integers(1, 900))
        out.append((T, h, fs * t, t))
    return out


@pytest.mark.parametrize("shape", _random_shapes(), ids=lambda s: "T%d_h%d_f%d_t%d" % s)
def test_random_shapes_full_oracle(shape):
    T, h, f, t = shape
    inp = inputs.make_custom(T, h, f, seed=T * 5 + h + f + t)
    check_full(run_fp8(to_gpu(inp), t), oracle.full(inp))


def test_weight_beyond_fp16_is_reported():
    """A weight fp16 cannot hold (|w| > 65504, fine in bf16) makes the fp16 copy of B infinite; the cast
    records MLP_ERR_RANGE instead of the step failing silently."""
    T, h, f, t = 128, 128, 512, 2
    host = inputs.make_custom(T, h, f, seed=45)
    host["B"][3, 7] = 1.0e5
    inp = to_gpu(host)
    out = block.alloc_outputs(T, h, f, mode=FP8)
    ws = binding.make_workspace_mode(T, h, f, t, FP8)
    block.forward(inp, t, out, ws, FP8)
    with pytest.raises(binding.MlpError) as err:
        binding.mlp_tp_check(ws)
    assert err.value.status == 9


def test_t_independence_and_determinism():
    """As in the bf16 modes: Z, H, H_lo, dA, dB, da, db do not depend on t bit for bit (the scales follow from
    statistics over whole tensors, not shards), Y and dX only through the shard-sum order, and a rerun
    (statistics by atomic max, copies on the side stream) gives the same bits."""
    T, h, f = 384, 512, 2048
    inp = to_gpu(inputs.make_custom(T, h, f, seed=5))
    outs = {t: run_fp8(inp, t) for t in (1, 2, 4, 8)}
    same = lambda a, b: torch.equal(a.view(torch.uint8), b.view(torch.uint8))  # noqa: E731
    for t in (2, 4, 8):
        for k in ("Z", "H", "H_lo", "dA", "dB", "da", "db"):
            assert same(outs[t][k], outs[1][k]), (k, t)
        for k in ("Y", "dX"):
            d = (outs[t][k].float() - outs[1][k].float()).abs()
            assert float(d.max()) <= 1e-2 * (1 + float(outs[1][k].float().abs().max())), (k, t)
    again = run_fp8(inp, 8)
    for k in again:
        assert same(again[k], outs[8][k]), k


def test_outputs_stay_inside_their_buffers():
    """Guard bands around every output and saved activation, with a ragged shape: the fp16 and e4m3 tiles'
    stores (32-byte rows for e4m3) are clipped at the tensors' edges."""
    T, h, f, t = 200, 192, 384, 3
    inp = to_gpu(inputs.make_custom(T, h, f, seed=4))
    shapes = {"Y": (T, h), "Z": (T, f), "H": (T, f), "H_lo": (T, f), "dX": (T, h), "dA": (h, f), "dB": (f, h),
              "da": (f,), "db": (h,)}
    dtypes = {"Z": torch.float32, "H": torch.float16, "H_lo": torch.uint8}
    pad = 4096
    bufs, out = {}, {}
    for k, s in shapes.items():
        n = int(np.prod(s))
        buf = torch.full((n + 2 * pad,), 0x5A, dtype=torch.uint8, device="cuda") if k == "H_lo" else \
            torch.full((n + 2 * pad,), -12345.0, dtype=dtypes.get(k, torch.bfloat16), device="cuda")
        bufs[k] = buf
        out[k] = buf[pad:pad + n].view(*s)
    ws = binding.make_workspace_mode(T, h, f, t, FP8)
    block.forward(inp, t, out, ws, FP8)
    block.backward(inp, t, out, ws, FP8)
    binding.mlp_tp_check(ws)
    for k, buf in bufs.items():
        n = int(np.prod(shapes[k]))
        head, tail = buf[:pad].cpu(), buf[pad + n:].cpu()
        assert torch.equal(head, torch.full_like(head, head[0])) and torch.equal(tail, torch.full_like(tail, head[0])), k
    out["H_lo"] = out["H_lo"].view(torch.float8_e4m3fn)
    check_full(out, oracle.full(inputs.make_custom(T, h, f, seed=4)))
