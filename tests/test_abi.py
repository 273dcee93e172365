"""The C-ABI library: it loads without a GPU, exports every symbol the
header declares, and rejects bad arguments on the host before touching the
device (CPU-only)."""
import ctypes
import os
import re

import pytest

from tensor_transformer_mlp_bias_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mlp_tp.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.lib()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mlp_tp_\w+)\s*\(", text)))


def test_header_declares_what_binding_wraps():
    assert header_functions() == sorted(binding.exported_symbols())


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in binding.STATUS.items():
        assert binding.mlp_tp_status_string(code) == name


def test_workspace_bytes(lib):
    n = binding.workspace_bytes(64, 256, 1024, 2)
    # header 256 + dH pair 2*64*1024*2 + da partials (one 256-row pair tile = two 128-row blocks,
    # 4 lane quadrants each, f fp32 column sums per quadrant) + room for the split pieces of the
    # shard-sum GEMMs' last wave (1 tile x t=2 shards, 256x256 fp32 each)
    assert n == 256 + 2 * 64 * 1024 * 2 + 2 * 4 * 1024 * 4 + 2 * 256 * 256 * 4
    assert binding.workspace_bytes(64, 256, 1000, 2) == 0   # f/t not a multiple of 64
    assert binding.workspace_bytes(64, 100, 1024, 2) == 0   # h not a multiple of 64
    assert binding.workspace_bytes(64, 256, 1024, 0) == 0   # t < 1
    assert binding.workspace_bytes(-1, 256, 1024, 2) == 0


def test_recompute_workspace_bytes(lib):
    T, h, f, t = 200, 192, 384, 6
    base = binding.workspace_bytes(T, h, f, t)
    rnd = lambda n: (n + 255) // 256 * 256  # noqa: E731
    # the ordinary workspace, then Z (fp32) and the H pair
    assert binding.recompute_workspace_bytes(T, h, f, t) == base + rnd(T * f * 4) + 2 * rnd(T * f * 2)
    assert binding.recompute_workspace_bytes(T, h, 100, t) == 0


FAKE = 1 << 20  # a 16-byte aligned fake address: validation must fail before any use


def call_fc1(lib, **kw):
    args = dict(X=FAKE, A=FAKE, a=FAKE, T=64, h=256, f=1024, t=2, Z=FAKE, H=FAKE, H_lo=FAKE, ws=FAKE * 2,
                ws_bytes=1 << 30, stream=None)
    args.update(kw)
    return lib.mlp_tp_fc1_forward(args["X"], args["A"], args["a"], args["T"], args["h"], args["f"], args["t"],
                                  args["Z"], args["H"], args["H_lo"], args["ws"], args["ws_bytes"], args["stream"])


@pytest.mark.parametrize("kw,status,needle", [
    (dict(X=None), 1, "X is NULL"),
    (dict(H=None), 1, "H is NULL"),
    (dict(H_lo=None), 1, "H_lo is NULL"),
    (dict(t=0), 1, "t=0"),
    (dict(T=-5), 1, "negative"),
    (dict(h=96), 2, "h=96"),
    (dict(f=1025), 2, "not divisible"),
    (dict(f=1024 + 64, t=2), 2, "multiple of 64"),
    (dict(A=FAKE + 8), 3, "A is not 16-byte aligned"),
    (dict(ws=None), 1, "workspace pointer is NULL"),
    (dict(ws=FAKE + 16), 3, "workspace is not 256-byte aligned"),
    (dict(ws_bytes=100), 4, "needs"),
])
def test_bad_arguments_are_rejected_on_the_host(lib, kw, status, needle):
    st = call_fc1(lib, **kw)
    assert st == status, binding.mlp_tp_last_error()
    assert needle in binding.mlp_tp_last_error()


def test_valid_arguments_without_a_gpu_report_the_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert call_fc1(lib) == 5  # MLP_ERR_UNSUPPORTED_DEVICE, nothing launched


def test_launch_counter_and_hooks_callable(lib):
    c0 = binding.mlp_tp_launch_count()
    binding.mlp_tp_set_wait_budget_ns(10)       # raised to the 1 ms floor
    binding.mlp_tp_set_wait_budget_ns(1_000_000_000)
    binding.mlp_tp_set_debug_flags(0)
    assert binding.mlp_tp_launch_count() == c0


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(64, 256, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        binding.mlp_tp_fc1_forward(x, x, x, 64, 256, 1024, 2, x, x, x, (FAKE, 1 << 30), stream=0)


def test_fp8_workspace_bytes(lib):
    """MLP_TP_FP8 adds its operand copies after the mode-independent
    workspace: W16 (fp16 B or A, 2·h·f), X16 and dY16 (2·T·h each), X8 and
    dY8 (T·h each), each rounded up to 256 bytes."""
    T, h, f, t = 200, 192, 384, 6
    rnd = lambda n: (n + 255) // 256 * 256  # noqa: E731
    extra = rnd(2 * h * f) + 2 * rnd(2 * T * h) + 2 * rnd(T * h)
    for mode in (binding.ACCURATE, binding.FAST_FC2_FORWARD, binding.FAST):
        assert binding.workspace_bytes_mode(T, h, f, t, mode) == binding.workspace_bytes(T, h, f, t)
        assert binding.recompute_workspace_bytes_mode(T, h, f, t, mode) == binding.recompute_workspace_bytes(T, h, f, t)
    assert binding.workspace_bytes_mode(T, h, f, t, binding.FP8) == binding.workspace_bytes(T, h, f, t) + extra
    assert (binding.recompute_workspace_bytes_mode(T, h, f, t, binding.FP8)
            == binding.recompute_workspace_bytes(T, h, f, t) + extra)
    assert binding.workspace_bytes_mode(T, h, f, t, 5) == 0
    assert binding.workspace_bytes_mode(T, h, 100, t, binding.FP8) == 0


def test_fp8_mode_checks_its_workspace(lib):
    T, h, f, t = 64, 256, 1024, 2
    small = binding.workspace_bytes(T, h, f, t)  # enough for every other mode
    st = lib.mlp_tp_forward(FAKE, FAKE, FAKE, FAKE, FAKE, T, h, f, t, binding.FP8, FAKE, FAKE, FAKE, FAKE,
                            FAKE * 2, small, None)
    assert st == 4 and "workspace" in binding.mlp_tp_last_error()
    st = lib.mlp_tp_fc2_backward_weight_fp8(FAKE, FAKE, FAKE, T, h, f, t, FAKE, None, FAKE * 2, small, None)
    assert st == 4
    # with enough workspace the call gets as far as the device check (no GPU
    # here; with one, fake addresses must never reach a launch)
    import torch
    if torch.cuda.is_available():
        return
    big = binding.workspace_bytes_mode(T, h, f, t, binding.FP8)
    st = lib.mlp_tp_backward(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, T, h, f, t, binding.FP8, FAKE, FAKE, None,
                             FAKE, None, FAKE * 2, big, None)
    assert st == 5


def test_precision_mode_is_validated(lib):
    for bad in (5, 7, -1):
        st = lib.mlp_tp_forward(FAKE, FAKE, FAKE, FAKE, FAKE, 64, 256, 1024, 2, bad, FAKE, FAKE, FAKE, FAKE,
                                FAKE * 2, 1 << 30, None)
        assert st == 1 and "precision mode" in binding.mlp_tp_last_error()


def test_accurate_mode_is_zero():
    """A caller that passes 0 (or zero-initialised options) gets the mode that
    meets the parity bar on every tested workload."""
    assert binding.ACCURATE == 0 and binding.FAST == binding.FAST_FC2_FORWARD | binding.FAST_FC1_BACKWARD_DATA
    text = open(HEADER).read()
    assert "MLP_TP_ACCURATE = 0" in text


C_CLIENT = r"""
/* A plain C99 client of the library: no CUDA headers, no torch. */
#include <stdio.h>
#include <string.h>
#include "mlp_tp.h"

int main(void) {
  size_t n = mlp_tp_workspace_bytes(64, 256, 1024, 2);
  if (n == 0) return 1;
  if (mlp_tp_workspace_bytes(64, 256, 1000, 3) != 0) return 2;          /* f not divisible by t */
  if (strcmp(mlp_tp_status_string(MLP_ERR_MISALIGNED), "MLP_ERR_MISALIGNED") != 0) return 3;
  /* NULL X is refused on the host, before any device work */
  mlp_status_t st = mlp_tp_fc1_forward(NULL, (void*)0x100000, (void*)0x100000, 64, 256, 1024, 2,
                                       (void*)0x100000, (void*)0x100000, (void*)0x100000,
                                       (void*)0x200000, (size_t)1 << 30, NULL);
  if (st != MLP_ERR_INVALID_ARG || strstr(mlp_tp_last_error(), "X") == NULL) return 4;
  printf("%zu\n", n);
  return 0;
}
"""


def test_header_is_plain_c_and_links_from_c(lib, tmp_path):
    """The header compiles as C99 and a C program links the library and
    calls it (host-side entry points only: no GPU here)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(binding.LIB_PATH)
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
           "-o", str(exe), "-L", libdir, "-l:" + os.path.basename(binding.LIB_PATH), "-Wl,-rpath," + libdir]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, (run.returncode, run.stderr)
    assert int(run.stdout.strip()) == binding.workspace_bytes(64, 256, 1024, 2)


# ------------------------------------------------------------------ cross-GPU entry points (host side)
def test_peer_buffer_sizes(lib):
    # [world][T/world][h] fp32 receive buffer; two uint32 per (128-row block, 256-column block) of a rank
    assert binding.peer_recv_bytes(4096, 4096, 8) == 4096 * 4096 * 4
    assert binding.peer_flag_bytes(4096, 4096, 8) == 2 * 4 * 16 * 4   # 512 rows per rank: 4 blocks x 16
    assert binding.peer_flag_bytes(4096, 4096, 1) == 2 * 32 * 16 * 4
    assert binding.peer_recv_bytes(333, 320, 1) == (333 * 320 * 4 + 255) // 256 * 256
    assert binding.peer_recv_bytes(100, 256, 3) == 0              # T not divisible by the ranks
    assert binding.peer_recv_bytes(64, 96, 1) == 0                # h not a multiple of 64
    assert binding.peer_flag_bytes(64, 256, 9) == 0               # more ranks than one NVLink group holds


def _fc2_peer(lib, peer, T=512, h=256, fs=128):
    import ctypes
    return lib.mlp_tp_fc2_forward_peer(FAKE, None, FAKE, T, h, fs, None if peer is None else ctypes.byref(peer),
                                       FAKE * 2, 1 << 30, None)


@pytest.mark.parametrize("kw,status,needle", [
    (None, 1, "peer descriptor is NULL"),
    (dict(world=9), 1, "world 9"),
    (dict(rank=2, world=2), 1, "rank 2"),
    (dict(world=3), 2, "do not split"),
    (dict(world=2, T=640), 2, "multiple of 128"),
    (dict(world=2, recv=[FAKE, None]), 1, "receive buffer 1 is NULL"),
    (dict(world=2, recv=[FAKE, FAKE + 4]), 3, "receive buffer 1 is not 16-byte aligned"),
    (dict(world=2, epoch=1, flags=None), 1, "flag block 0 is NULL"),
    (dict(reserved=5), 1, "reserved"),
])
def test_peer_descriptor_is_validated_on_the_host(lib, kw, status, needle):
    if kw is None:
        st = _fc2_peer(lib, None)
    else:
        world = kw.get("world", 1)
        recv = kw.get("recv", [FAKE] * world)
        flags = kw.get("flags", [FAKE] * world)
        peer = binding.Peer()
        peer.rank, peer.world, peer.epoch = kw.get("rank", 0), world, kw.get("epoch", 0)
        peer.reserved = kw.get("reserved", 0)
        for o in range(min(world, binding.MAX_WORLD)):
            peer.recv[o] = recv[o]
            peer.flags[o] = flags[o] if flags is not None else None
        st = _fc2_peer(lib, peer, T=kw.get("T", 512))
    assert st == status, binding.mlp_tp_last_error()
    assert needle in binding.mlp_tp_last_error()


def test_make_peer_checks_its_table():
    with pytest.raises(ValueError):
        binding.make_peer(2, 2, [FAKE, FAKE])
    with pytest.raises(ValueError):
        binding.make_peer(0, 2, [FAKE])
    p = binding.make_peer(1, 2, [FAKE, FAKE * 2], [FAKE * 3, FAKE * 4], 7)
    assert (p.rank, p.world, p.epoch) == (1, 2, 7) and p.recv[1] == FAKE * 2 and p.flags[0] == FAKE * 3
