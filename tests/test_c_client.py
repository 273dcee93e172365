"""The C-ABI from a C++ host program on the GPU, with no Python or torch in
the process: cudaMalloc'd buffers, mlp_tp_forward, mlp_tp_backward and
mlp_tp_check, built here with g++ against include/mlp_tp.h and the CUDA
runtime.  The seeded inputs go in as a raw bf16 file; the outputs come back
as raw files and are checked against the oracle with the parity bar.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

from oracle import mlp_oracle as oracle
from tensor_transformer_mlp_bias_b200 import binding, inputs
from tests.parity_util import assert_close

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = "/usr/local/cuda"

CLIENT = r"""
#include <cuda_runtime.h>
#include <cstdio>
#include <cstdlib>
#include <cstdint>
#include <vector>
#include "mlp_tp.h"

#define CK(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) { \
  std::fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_)); return 10; } } while (0)
#define MK(x) do { mlp_status_t s_ = (x); if (s_ != MLP_OK) { \
  std::fprintf(stderr, "%s: %s %s\n", #x, mlp_tp_status_string(s_), mlp_tp_last_error()); return 11; } } while (0)

static void* dev_from(FILE* f, size_t bytes) {
  std::vector<unsigned char> h(bytes);
  if (std::fread(h.data(), 1, bytes, f) != bytes) return nullptr;
  void* d = nullptr;
  if (cudaMalloc(&d, bytes) != cudaSuccess) return nullptr;
  if (cudaMemcpy(d, h.data(), bytes, cudaMemcpyHostToDevice) != cudaSuccess) return nullptr;
  return d;
}

static int to_file(const char* path, const void* d, size_t bytes) {
  std::vector<unsigned char> h(bytes);
  if (cudaMemcpy(h.data(), d, bytes, cudaMemcpyDeviceToHost) != cudaSuccess) return 1;
  FILE* f = std::fopen(path, "wb");
  if (!f) return 1;
  std::fwrite(h.data(), 1, bytes, f);
  std::fclose(f);
  return 0;
}

int main(int argc, char** argv) {
  if (argc != 8) return 2;
  const int mode = std::atoi(argv[7]);  // MLP_TP_ACCURATE, or MLP_TP_FP8 (H then holds fp16 values)
  const int64_t T = std::atoll(argv[1]), h = std::atoll(argv[2]), f = std::atoll(argv[3]);
  const int32_t t = std::atoi(argv[4]);
  const char* in_path = argv[5];
  const char* out_dir = argv[6];
  FILE* fin = std::fopen(in_path, "rb");
  if (!fin) return 3;
  const size_t b2 = 2;  // bf16
  void* X = dev_from(fin, T * h * b2);
  void* A = dev_from(fin, h * f * b2);
  void* a = dev_from(fin, f * b2);
  void* B = dev_from(fin, f * h * b2);
  void* b = dev_from(fin, h * b2);
  void* dY = dev_from(fin, T * h * b2);
  std::fclose(fin);
  if (!X || !A || !a || !B || !b || !dY) return 4;
  void *Y, *Z, *H, *H_lo, *dX, *dA, *da, *dB, *db, *ws;
  CK(cudaMalloc(&Y, T * h * b2));
  CK(cudaMalloc(&Z, T * f * 4));
  CK(cudaMalloc(&H, T * f * b2));
  CK(cudaMalloc(&H_lo, T * f * b2));
  CK(cudaMalloc(&dX, T * h * b2));
  CK(cudaMalloc(&dA, h * f * b2));
  CK(cudaMalloc(&da, f * b2));
  CK(cudaMalloc(&dB, f * h * b2));
  CK(cudaMalloc(&db, h * b2));
  const size_t ws_bytes = mlp_tp_workspace_bytes_mode(T, h, f, t, mode);
  if (ws_bytes == 0) return 5;
  CK(cudaMalloc(&ws, ws_bytes));
  CK(cudaMemset(ws, 0, ws_bytes));
  cudaStream_t s;
  CK(cudaStreamCreate(&s));
  MK(mlp_tp_forward(X, A, a, B, b, T, h, f, t, mode, Y, Z, H, H_lo, ws, ws_bytes, s));
  MK(mlp_tp_backward(dY, X, A, B, Z, H, H_lo, T, h, f, t, mode, dX, dA, da, dB, db, ws, ws_bytes, s));
  MK(mlp_tp_check(ws, s));
  char p[4096];
  const char* names[] = {"Y", "Z", "H", "dX", "dA", "da", "dB", "db"};
  void* ptrs[] = {Y, Z, H, dX, dA, da, dB, db};
  const size_t sizes[] = {(size_t)(T * h * b2), (size_t)(T * f * 4), (size_t)(T * f * b2), (size_t)(T * h * b2),
                          (size_t)(h * f * b2), (size_t)(f * b2), (size_t)(f * h * b2), (size_t)(h * b2)};
  for (int i = 0; i < 8; ++i) {
    std::snprintf(p, sizeof(p), "%s/%s.bin", out_dir, names[i]);
    if (to_file(p, ptrs[i], sizes[i])) return 6;
  }
  std::printf("launches %llu\n", (unsigned long long)mlp_tp_launch_count());
  return 0;
}
"""


def _bf16_bytes(x: torch.Tensor) -> bytes:
    return x.contiguous().view(torch.int16).numpy().tobytes()


def _load(path, shape, f32=False):
    raw = np.fromfile(path, dtype=np.float32 if f32 else np.uint16)
    if f32:
        return raw.reshape(shape).astype(np.float64)
    return (raw.astype(np.uint32) << 16).view(np.float32).reshape(shape).astype(np.float64)


@pytest.mark.parametrize("mode", [0, 4], ids=["accurate", "fp8"])
def test_cpp_client_runs_the_block_through_the_c_abi(tmp_path, mode):
    gxx = shutil.which("g++")
    if gxx is None or not os.path.exists(os.path.join(CUDA, "include", "cuda_runtime.h")):
        pytest.skip("g++ or the CUDA headers are not available")
    binding.lib()  # builds nothing; fails loudly if the library is missing
    src = tmp_path / "client.cpp"
    src.write_text(CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(binding.LIB_PATH)
    cmd = [gxx, "-std=c++17", "-O1", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), str(src), "-o", str(exe),
           "-L", libdir, "-l:" + os.path.basename(binding.LIB_PATH), "-Wl,-rpath," + libdir,
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-Wl,-rpath," + os.path.join(CUDA, "lib64")]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr

    T, h, f, t = 333, 320, 1280, 5
    inp = inputs.make_custom(T, h, f, seed=61)
    blob = tmp_path / "in.bin"
    with open(blob, "wb") as fh:
        for k in ("X", "A", "a", "B", "b", "dY"):
            fh.write(_bf16_bytes(inp[k]))
    out_dir = tmp_path / "out"
    out_dir.mkdir()
    run = subprocess.run([str(exe), str(T), str(h), str(f), str(t), str(blob), str(out_dir), str(mode)],
                         capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, (run.returncode, run.stdout, run.stderr)
    assert int(run.stdout.split()[-1]) > 0  # the library's own kernels ran

    ref = oracle.full(inp)
    shapes = {"Y": (T, h), "Z": (T, f), "H": (T, f), "dX": (T, h), "dA": (h, f), "da": (f,), "dB": (f, h),
              "db": (h,)}
    for k, shp in shapes.items():
        if k == "H" and mode == 4:  # the fp8 mode's H is fp16 (its e4m3 residual stays on the device)
            got = np.fromfile(out_dir / "H.bin", dtype=np.float16).reshape(shp).astype(np.float64)
        else:
            got = _load(out_dir / f"{k}.bin", shp, f32=(k == "Z"))
        assert_close(k + " (C++ client)", got, ref[k])
