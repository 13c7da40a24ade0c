"""The C-ABI library: it builds, loads, exports every symbol include/moe.h
declares, and validates arguments on the host.  No compute call is made (no
GPU is needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O
from sparse_mixture_experts_gating_b200 import _build, _lib

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe.h")


@pytest.fixture(scope="module")
def L():
    _build.build()
    return _lib.lib()


def declared_functions():
    src = open(HEADER).read()
    return re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src, flags=re.M)


def test_header_declares_the_boundary():
    names = declared_functions()
    assert {"moe_create", "moe_forward", "moe_destroy", "moe_workspace_bytes", "moe_status"} <= set(names)
    assert set(names) == set(_lib.SIGNATURES), "binding and header disagree"


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def _create(L, *args):
    h = ctypes.c_void_p()
    rc = L.moe_create(*args, ctypes.byref(h))
    return rc, h


def test_create_validates_arguments(L):
    ok, h = _create(L, 8, 2, 4096, 14336, 1, 1, 0.0, 1)
    assert ok == _lib.MOE_OK and h.value
    L.moe_destroy(h)
    bad = [
        (0, 1, 64, 64, 0, 1, 0.0, 1),      # no experts
        (257, 1, 64, 64, 0, 1, 0.0, 1),    # too many experts
        (4, 5, 64, 64, 0, 1, 0.0, 1),      # k > E
        (16, 9, 64, 64, 0, 1, 0.0, 1),     # k > 8
        (4, 0, 64, 64, 0, 1, 0.0, 1),      # k = 0
        (4, 2, 0, 64, 0, 1, 0.0, 1),       # d = 0
        (4, 2, 64, 64, 2, 1, 0.0, 1),      # unknown act
        (4, 2, 64, 64, 0, 2, 0.0, 1),      # unknown gate
        (4, 2, 64, 64, 0, 1, 0.0, 7),      # unknown dtype
        (4, 2, 64, 64, 0, 1, float("nan"), 1),
    ]
    for args in bad:
        rc, h = _create(L, *args)
        assert rc == _lib.MOE_ERR_INVALID_ARG, args
        assert h.value is None
        assert L.moe_last_error().decode().startswith("moe_create")
    rc, _ = _create(L, 4, 2, 60, 64, 0, 1, 0.0, 1)  # bf16 rows must be 16-byte multiples
    assert rc == _lib.MOE_ERR_UNSUPPORTED
    rc, h = _create(L, 4, 2, 60, 62, 0, 1, 0.0, 0)  # fp32 accepts any width
    assert rc == _lib.MOE_OK
    L.moe_destroy(h)


def test_capacity_matches_the_oracle(L):
    rng = np.random.default_rng(3)
    for _ in range(300):
        E = int(rng.integers(1, 257)); k = int(rng.integers(1, min(E, 8) + 1))
        cf = float(rng.choice([0.0, -1.0, 1.0, 1.25, 2.0, rng.uniform(0.01, 4.0)]))
        T = int(rng.integers(0, 100000))
        rc, h = _create(L, E, k, 64, 64, 0, 1, cf, 1)
        assert rc == 0
        c = L.moe_capacity(h, T)
        ref = O.expert_capacity(cf, T, k, E)
        assert (None if c < 0 else c) == ref, (E, k, cf, T)
        L.moe_destroy(h)


def test_workspace_and_forward_validation_without_gpu(L):
    rc, h = _create(L, 64, 1, 768, 3072, 0, 0, 1.25, 1)
    assert rc == 0
    ws = L.moe_workspace_bytes(h, 8192)
    # Xp + Hp + routing tables at least; capacity 160 bounds the sorted rows
    assert ws >= 2 * 8192 * (768 + 3072)
    assert L.moe_workspace_bytes(h, -1) == 0
    assert L.moe_workspace_bytes(None, 16) == 0
    p = ctypes.c_void_p(256)
    # NULL handle, negative T, NULL statistics outputs: rejected before any CUDA call
    assert L.moe_forward(None, 4, p, p, None, p, None, p, p, p, p, p, p, p, 1 << 30, None, None) == 1
    assert L.moe_forward(h, -1, p, p, None, p, None, p, p, p, p, p, p, p, 1 << 30, None, None) == 1
    assert L.moe_forward(h, 4, p, p, None, p, None, p, p, None, p, p, p, p, 1 << 30, None, None) == 1
    # W3 given for a ReLU layer
    assert L.moe_forward(h, 4, p, p, None, p, p, p, p, p, p, p, p, p, 1 << 30, None, None) == 1
    # workspace too small / misaligned
    assert L.moe_forward(h, 4, p, p, None, p, None, p, p, p, p, p, p, p, 16, None, None) == 1
    assert L.moe_forward(h, 4, p, p, None, p, None, p, p, p, p, p, p, ctypes.c_void_p(272), 1 << 30,
                         None, None) == 1
    assert "workspace" in L.moe_last_error().decode()
    L.moe_destroy(h)
    assert L.moe_destroy(None) == 0


def test_shared_experts_and_balance_losses_validate_arguments(L):
    rc, h = _create(L, 8, 2, 64, 64, 1, 1, 0.0, 1)
    assert rc == 0
    ws0 = L.moe_workspace_bytes(h, 100)
    for bad in (-1, 9):
        assert L.moe_set_shared_experts(h, bad) == _lib.MOE_ERR_INVALID_ARG
    assert L.moe_set_shared_experts(None, 1) == _lib.MOE_ERR_INVALID_ARG
    assert L.moe_set_shared_experts(h, 2) == 0
    # two shared experts add 2 * T rows to every expert-sorted buffer
    assert L.moe_workspace_bytes(h, 100) >= ws0 + 2 * 100 * (64 + 64) * 2
    rc2, h2 = _create(L, 255, 2, 64, 64, 1, 1, 0.0, 1)
    assert L.moe_set_shared_experts(h2, 2) == _lib.MOE_ERR_INVALID_ARG  # E + n_shared > 256
    assert L.moe_set_shared_experts(h2, 1) == 0
    p = ctypes.c_void_p(256)
    assert L.moe_balance_losses(None, 4, p, p, None) == _lib.MOE_ERR_INVALID_ARG
    assert L.moe_balance_losses(h, -1, p, p, None) == _lib.MOE_ERR_INVALID_ARG
    assert L.moe_balance_losses(h, 4, p, None, None) == _lib.MOE_ERR_INVALID_ARG
    assert L.moe_balance_losses(h, 4, None, p, None) == _lib.MOE_ERR_INVALID_ARG
    L.moe_destroy(h)
    L.moe_destroy(h2)


def test_workspace_sizing_is_defined_for_every_batch_size(L):
    """Host-only sizing (no GPU): every T from 0 up, several layer shapes, every
    hidden precision (the automatic one across its switch to fp16); sizes
    never shrink as T grows."""
    shapes = [(8, 2, 4096, 14336, 1, 1, 0.0, 1), (64, 1, 768, 3072, 0, 0, 1.25, 1),
              (128, 4, 2048, 768, 1, 1, 2.0, 1), (4, 2, 32, 64, 0, 1, 0.0, 0), (256, 8, 64, 64, 0, 0, 0.5, 1),
              (3, 2, 1032, 1160, 1, 1, 0.0, 1)]
    for i, args in enumerate(shapes):
        rc, h = _create(L, *args)
        assert rc == 0
        ns = min(i % 3, 256 - args[0])
        assert L.moe_set_shared_experts(h, ns) == 0
        E, k = args[0], args[1]
        t_auto = 1024 * (E + ns) // (k + ns)  # near where the automatic mode turns to fp16
        extra = sorted({t for t in range(t_auto - 3, t_auto + 4) if t > 0} | {511, 512, 513, 2047, 2048, 2049,
                                                                               8192, 16384})
        for mode in (0, 1, 2, 3):
            assert L.moe_set_hidden_precision(h, mode) == 0
            prev = 0
            for T in list(range(0, 300)) + extra:
                n = L.moe_workspace_bytes(h, T)
                assert n >= prev and n % 256 == 0, (args, mode, T, n)
                prev = n
        L.moe_destroy(h)


def test_4bit_workspace_never_shrinks_as_T_grows(L):
    """moe_workspace_bytes_w4 across the switch from the few-row products
    (T <= 16, fp32 partials of the first projection) to the grouped GEMM."""
    shapes = [(8, 2, 4096, 14336, 1, 1, 0.0, 1), (64, 1, 768, 3072, 0, 0, 1.25, 1),
              (16, 4, 1024, 2048, 1, 1, 0.0, 1), (2, 2, 384, 640, 0, 0, 0.0, 1)]
    for i, args in enumerate(shapes):
        rc, h = _create(L, *args)
        assert rc == 0
        assert L.moe_set_shared_experts(h, i % 2) == 0
        prev = 0
        for T in list(range(0, 300)) + [511, 512, 513, 4096]:
            n = L.moe_workspace_bytes_w4(h, T)
            assert n >= prev and n % 256 == 0, (args, T, n)
            prev = n
        L.moe_destroy(h)


def test_automatic_hidden_mode_adds_the_fp16_weight_image_at_1024_rows_per_expert(L):
    """The automatic mode holds the hidden activation in fp16 (and reserves the
    fp16 image of W2) from 1024 rows per expert group on: for 8 experts, top-2,
    dropless, that is T = 4096."""
    rc, h = _create(L, 8, 2, 4096, 14336, 1, 1, 0.0, 1)
    assert rc == 0
    image = 8 * 4096 * 14336 * 2
    assert L.moe_set_hidden_precision(h, 3) == 0
    below, at = L.moe_workspace_bytes(h, 4095), L.moe_workspace_bytes(h, 4096)
    assert at - below >= image
    assert L.moe_set_hidden_precision(h, 2) == 0  # forced fp16: the image at any T
    assert L.moe_workspace_bytes(h, 1) >= image
    assert L.moe_set_hidden_precision(h, 0) == 0  # forced pair: no image
    assert L.moe_workspace_bytes(h, 4096) < at
    assert L.moe_set_hidden_precision(h, 4) == _lib.MOE_ERR_INVALID_ARG
    L.moe_destroy(h)


def test_static_scratch_limit_stated_in_the_header_holds(L):
    """The header's example limit of moe_forward_static matches the sizing."""
    m = re.search(r"d_ff 14336 SwiGLU layer up to T = (\d+)\)", open(HEADER).read())
    assert m, "example limit not found in include/moe.h"
    stated = int(m.group(1))
    rc, h = _create(L, 8, 2, 4096, 14336, 1, 1, 0.0, 1)
    assert rc == 0
    lim = 32 << 20
    assert L.moe_workspace_bytes(h, stated) <= lim < L.moe_workspace_bytes(h, stated + 1)
    L.moe_destroy(h)


def test_backward_validates_arguments_without_gpu(L):
    rc, h = _create(L, 8, 2, 64, 64, 1, 1, 0.0, 1)  # SwiGLU
    assert rc == 0
    prev = 0
    for T in range(0, 300):
        n = L.moe_backward_workspace_bytes(h, T)
        assert n >= prev and n % 256 == 0
        prev = n
    assert L.moe_backward_workspace_bytes(None, 4) == 0 and L.moe_backward_workspace_bytes(h, -1) == 0
    p = ctypes.c_void_p(256)
    big = 1 << 40

    def call(hh=h, T=4, W3=p, dW3=p, ws=p, ws_n=big, bw=p, bw_n=big, x=p):
        return L.moe_backward(hh, T, x, p, None, p, W3, p, p, 0.0, 0.0, p, p, None, p, dW3, p, ws, ws_n, bw,
                              bw_n, None)

    assert call(hh=None) == _lib.MOE_ERR_INVALID_ARG
    assert call(T=-1) == _lib.MOE_ERR_INVALID_ARG
    assert call(W3=None) == _lib.MOE_ERR_INVALID_ARG   # SwiGLU needs W3 ...
    assert call(dW3=None) == _lib.MOE_ERR_INVALID_ARG  # ... and dW3
    assert call(x=None) == _lib.MOE_ERR_INVALID_ARG
    assert call(ws_n=16) == _lib.MOE_ERR_INVALID_ARG
    assert "forward workspace" in L.moe_last_error().decode()
    assert call(bw_n=16) == _lib.MOE_ERR_INVALID_ARG
    assert "backward workspace" in L.moe_last_error().decode()
    assert call(bw=ctypes.c_void_p(272)) == _lib.MOE_ERR_INVALID_ARG
    L.moe_destroy(h)


def test_header_compiles_and_links_as_plain_c(L, tmp_path):
    """A C program (not C++) includes include/moe.h, links the library and
    calls the host-only entry points."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_moe.c"
    src.write_text(r"""
#include <stdio.h>
#include "moe.h"
int main(void) {
  moe_handle h = 0;
  if (moe_create(64, 1, 768, 3072, MOE_ACT_RELU, MOE_GATE_SWITCH, 1.25, MOE_BF16, &h) != MOE_OK) return 1;
  if (moe_capacity(h, 8192) != 160) return 2;
  if (moe_workspace_bytes(h, 8192) == 0 || moe_backward_workspace_bytes(h, 8192) == 0) return 3;
  if (moe_forward(NULL, 1, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0) != MOE_ERR_INVALID_ARG) return 4;
  if (moe_destroy(h) != MOE_OK) return 5;
  printf("ok\n");
  return 0;
}
""")
    lib_dir = os.path.dirname(L._name)
    exe = tmp_path / "use_moe"
    inc = os.path.dirname(HEADER)
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", "-I", inc, str(src), "-o", str(exe), "-L", lib_dir,
                        "-l:" + os.path.basename(L._name), "-Wl,-rpath," + lib_dir], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True)
    assert run.returncode == 0 and run.stdout.strip() == "ok", (run.returncode, run.stdout, run.stderr)


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    """No CPU fallback: with the library absent the binding raises instead of
    computing anything."""
    monkeypatch.setattr(_lib, "_LIB", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libmoe_b200.so"))
    with pytest.raises(ImportError, match="no CPU fallback"):
        _lib.lib()


def test_product_path_never_imports_the_oracle():
    """The package (binding, layer, workloads, build) and bench.py's timed arm
    reference the oracle nowhere; only tests, smoke() and the CPU baseline do."""
    pkg = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                       "sparse_mixture_experts_gating_b200")
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(root, f), encoding="utf-8").read()
                assert "import oracle" not in src and "from oracle" not in src, f
