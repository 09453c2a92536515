"""The oracle's Philox-4x32-10 pinned bit for bit against cuRAND's device
Philox4_32_10 generator (an implementation written by others from the same
paper: Salmon, Moraes, Dror, Shaw, SC'11, "Parallel Random Numbers: As Easy as
1, 2, 3").  Both the oracle and the library were written here from that paper;
a constant or round mistaken the same way in both would pass their mutual
comparison, but not this one.

Counter mapping (cuRAND's documented initialisation): the 64-bit seed is the
key (low word first), the subsequence selects the upper two counter words and
offset / 4 the lower two; curand4 returns the four words of that counter.
So the oracle's counter (c0, c1, c2, c3) is subsequence = c2 | c3 << 32,
offset = 4 (c0 | c1 << 32).  The probe is compiled from tests/cuda at test time."""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

from oracle.philox import philox4x32_10_np, seed_key

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def curand_lib(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("curand") / "libcurand_philox.so")
    nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-shared", "-Xcompiler", "-fPIC",
                    os.path.join(HERE, "cuda", "curand_philox.cu"), "-o", out], check=True)
    lib = ctypes.CDLL(out)
    lib.curand_philox_words.restype = ctypes.c_int
    lib.curand_philox_words.argtypes = [ctypes.c_ulonglong, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                        ctypes.c_void_p, ctypes.c_void_p]
    return lib


def _curand_words(lib, seed, c0, c1, c2, c3):
    sub = torch.from_numpy((c2.astype(np.uint64) | (c3.astype(np.uint64) << np.uint64(32))).view(np.int64)).cuda()
    off = torch.from_numpy((np.uint64(4) * (c0.astype(np.uint64) | (c1.astype(np.uint64) << np.uint64(32))))
                           .view(np.int64)).cuda()
    n = c0.shape[0]
    out = torch.empty((n, 4), dtype=torch.int32, device="cuda")
    rc = lib.curand_philox_words(seed, sub.data_ptr(), off.data_ptr(), n, out.data_ptr(),
                                 torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("seed", [0, 7, 1234, 0x123456789ABCDEF0, 2**64 - 1])
def test_oracle_philox_equals_curand(curand_lib, seed):
    rng = np.random.default_rng(seed % 1000)
    n = 100_000
    c0 = rng.integers(0, 2**32, n, dtype=np.uint64)
    c1 = rng.integers(0, 2**30, n, dtype=np.uint64)       # 4 (c0 | c1 << 32) must fit in 64 bits
    c2 = rng.integers(0, 2**32, n, dtype=np.uint64)
    c3 = rng.integers(0, 2**32, n, dtype=np.uint64)
    # the counters the method draws: (position, step, block, request)
    c0[:256], c1[:256], c2[:256], c3[:256] = np.arange(256), 12, 3, 1
    c0[256:512], c1[256:512], c2[256:512], c3[256:512] = np.arange(256), 0, 0, 0
    got = _curand_words(curand_lib, seed, c0, c1, c2, c3)
    k0, k1 = seed_key(seed)
    ref = np.stack(philox4x32_10_np(c0, c1, c2, c3, k0, k1), axis=1)
    bad = np.nonzero((got != ref).any(axis=1))[0]
    assert bad.size == 0, (f"{bad.size} of {n} counters differ; first: counter "
                           f"{[int(c[bad[0]]) for c in (c0, c1, c2, c3)]} cuRAND {got[bad[0]]} oracle {ref[bad[0]]}")
