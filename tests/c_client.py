"""Build and drive tests/c/awq_client.c, the plain C client of the library (no torch)."""
import os
import shutil
import subprocess
import struct

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SOURCE = os.path.join(ROOT, "tests", "c", "awq_client.c")
PKG = os.path.join(ROOT, "post_quantization_column_b200")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def compiler():
    return shutil.which("gcc") or shutil.which("cc")


def build(out_dir: str) -> str:
    """Compile the client as C99 against include/awq_search.h, libawqsearch.so and the
    CUDA runtime; returns the executable's path."""
    exe = os.path.join(out_dir, "awq_client")
    cmd = [compiler(), "-std=c99", "-O2", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), SOURCE, "-o", exe,
           "-L", PKG, "-lawqsearch", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           "-Wl,-rpath," + PKG, "-Wl,-rpath," + os.path.join(CUDA, "lib64")]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return exe


def write_input(path: str, X: np.ndarray, W: np.ndarray, group: int, n_grid: int, dtype: int) -> None:
    """X, W as raw little-endian arrays (uint16 bf16 bit patterns or float32)."""
    M, K = X.shape
    N = W.shape[1]
    with open(path, "wb") as f:
        f.write(struct.pack("<qqqiii", M, K, N, group, n_grid, dtype))
        f.write(np.ascontiguousarray(X).tobytes())
        f.write(np.ascontiguousarray(W).tobytes())


def read_output(path: str, K: int, N: int, group: int, n_grid: int):
    """Three records (status, scales, codes, steps, zeros, losses, best) of the client's calls."""
    sizes = [("scales", np.float32, (K,)), ("codes", np.int32, (K, N // 8)),
             ("steps", np.uint16, (K // group, N)), ("zeros", np.uint16, (K // group, N)),
             ("losses", np.float32, (n_grid,)), ("best", np.int32, (1,))]
    out = []
    with open(path, "rb") as f:
        for _ in range(3):
            rec = {"status": struct.unpack("<i", f.read(4))[0]}
            for name, dt, shape in sizes:
                n = int(np.prod(shape)) * np.dtype(dt).itemsize
                rec[name] = np.frombuffer(f.read(n), dtype=dt).reshape(shape)
            out.append(rec)
    return out
