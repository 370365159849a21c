"""The C ABI library loads, exports every function include/moe.h declares, and
rejects invalid arguments on the host (no GPU needed: nothing is launched)."""

import ctypes
import os
import re
import subprocess

import pytest

import sparse_mixture_experts_06_b200 as moe

ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))
HEADER = os.path.join(ROOT, "include", "moe.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("moe_router_topk", "moe_permute", "moe_expert_ffn", "moe_layer_forward"):
        assert required in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", moe.lib_path], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    # and nothing else leaks out of the shared object
    assert all(e.startswith("moe_") for e in exported), sorted(e for e in exported if not e.startswith("moe_"))
    for n in declared_functions():
        assert hasattr(moe.lib, n)


def test_version_and_error_string():
    assert "sm_100a" in moe.moe_version()
    assert isinstance(moe.moe_last_error_string(), str)


def _sz(T, d, f, E, k, dt):
    n = T * k
    a = lambda b: (b + 255) // 256 * 256  # noqa: E731
    esz = 2 if dt == moe.MOE_BF16 else 4
    # idx, w, perm, inv; offsets; x_perm (bf16); h; obuf; 4 GEMM tile counters; the combine's arrival
    # counters (one per token and 128 output columns); chunk bases of the permutation (E per 64
    # assignments)
    return (a(4 * n) * 4 + a(4 * (E + 1)) + (a(n * d * 2) if dt == moe.MOE_BF16 else 0)
            + a(n * f * esz) + a(n * d * 4) + a(4 * 4) + a(4 * T * ((d + 127) // 128))
            + a(4 * E * ((n + 63) // 64)))


@pytest.mark.parametrize("shape", [(4096, 4096, 14336, 8, 2), (32, 4096, 14336, 8, 2), (16, 64, 128, 8, 2),
                                   (1, 8, 8, 1, 1), (37, 72, 136, 8, 2)])
@pytest.mark.parametrize("dt", [0, 1])
def test_workspace_size(shape, dt):
    assert moe.moe_workspace_size(*shape, dt) == _sz(*shape, dt)


@pytest.mark.parametrize("bad", [dict(T=-1), dict(d=0), dict(d=12), dict(f=100), dict(E=0), dict(E=65),
                                 dict(k=0), dict(k=10, E=9), dict(dt=7)])
def test_workspace_size_invalid_is_zero(bad):
    a = dict(T=16, d=64, f=128, E=8, k=2, dt=0)
    a.update(bad)
    assert moe.moe_workspace_size(a["T"], a["d"], a["f"], a["E"], a["k"], a["dt"]) == 0


def call_router(**kw):
    a = dict(x=16, Wg=16, T=4, d=64, E=8, k=2, dt=0, idx=16, w=16)
    a.update(kw)
    P = ctypes.c_void_p
    return moe.lib.moe_router_topk(P(a["x"]), P(a["Wg"]), a["T"], a["d"], a["E"], a["k"], a["dt"], P(a["idx"]),
                                   P(a["w"]), None)


def test_router_rejects_invalid_arguments():
    assert call_router(x=0) == 1 and "x is NULL" in moe.moe_last_error_string()
    assert call_router(x=8) == 1 and "aligned" in moe.moe_last_error_string()
    assert call_router(Wg=0) == 1
    assert call_router(idx=0) == 1
    assert call_router(T=-3) == 1
    assert call_router(E=0) == 1
    assert call_router(k=3, E=2) == 1
    assert call_router(k=17, E=16) == 1         # k > E
    assert call_router(E=65, k=2) == 1          # more experts than the GPU path holds
    assert call_router(d=60) == 1
    assert call_router(dt=3) == 1
    # T = 0 is a no-op (nothing to launch), even with null pointers
    assert call_router(T=0, x=0, Wg=0, idx=0, w=0) == 0


def test_permute_rejects_invalid_arguments():
    P = ctypes.c_void_p
    f = moe.lib.moe_permute
    assert f(P(16), 4, 8, 2, None, P(16), P(16), None) == 1   # offsets NULL
    assert f(None, 4, 8, 2, P(16), P(16), P(16), None) == 1   # topk_idx NULL
    assert f(P(16), -1, 8, 2, P(16), P(16), P(16), None) == 1
    assert f(P(16), 4, 8, 9, P(16), P(16), P(16), None) == 1


def test_layer_rejects_invalid_arguments():
    P = ctypes.c_void_p
    ex = moe.lib.moe_layer_forward_ex
    # A valid argument list with fake pointers; every variant below breaks one
    # rule, so the call returns before anything is launched.  (The valid list
    # itself is never called.)
    args = [P(16)] * 5 + [None, 16, 64, 128, 8, 2, 0, P(256), 10 ** 9, P(512), None]
    bad = list(args)
    bad[12] = None                  # workspace NULL
    assert ex(*bad) == 3
    bad = list(args)
    bad[13] = 1000                  # workspace too small
    assert ex(*bad) == 3 and "workspace" in moe.moe_last_error_string()
    bad = list(args)
    bad[14] = P(16)                 # y aliases x
    assert ex(*bad) == 1
    bad = list(args)
    bad[8] = 100                    # f not a multiple of 8
    assert ex(*bad) == 1
    lf = moe.lib.moe_layer_forward
    assert lf(P(16), P(16), P(16), P(16), P(16), 4, 64, 128, 8, 0, P(512), None) == 1
    ffn = moe.lib.moe_expert_ffn
    assert ffn(P(16), P(16), P(16), P(16), None, P(16), P(16), P(16), 4, 64, 128, 8, 2, 0, P(256), 10 ** 9,
               P(512), None) == 1   # offsets NULL


def test_host_layer_rejects_invalid_arguments():
    """moe_layer_forward_host: argument errors are reported before any CUDA
    call (fake pointers; the valid list itself is never called)."""
    P = ctypes.c_void_p
    f = moe.lib.moe_layer_forward_host
    args = [P(8)] + [P(16)] * 4 + [16, 64, 128, 8, 2, P(8), 2, 0, None]
    bad = list(args); bad[0] = None                            # x_host NULL
    assert f(*bad) == 1 and "x_host" in moe.moe_last_error_string()
    bad = list(args); bad[10] = None                           # y_host NULL
    assert f(*bad) == 1 and "y_host" in moe.moe_last_error_string()
    bad = list(args); bad[11] = 0                              # no chunks
    assert f(*bad) == 1 and "chunks" in moe.moe_last_error_string()
    bad = list(args); bad[2] = P(24)                           # W1 not 16-byte aligned
    assert f(*bad) == 1 and "aligned" in moe.moe_last_error_string()
    bad = list(args); bad[9] = 9                               # k > E
    assert f(*bad) == 1
    bad = list(args); bad[12] = 6                              # unknown flag bits
    assert f(*bad) == 1 and "flags" in moe.moe_last_error_string()
    bad = list(args); bad[5] = 0; bad[0] = None; bad[10] = None  # T = 0: a no-op
    assert f(*bad) == 0


def test_stack_rejects_invalid_arguments():
    P = ctypes.c_void_p
    arr = (ctypes.c_void_p * 2)(16, 16)
    nul = (ctypes.c_void_p * 2)(16, 0)
    f = moe.lib.moe_stack_forward
    base = [P(16), arr, arr, arr, arr, 2, 4, 64, 128, 8, 2, 0, P(256), P(512), 10 ** 9, P(768), None]
    bad = list(base); bad[5] = 0
    assert f(*bad) == 1                                   # L < 1
    bad = list(base); bad[1] = None
    assert f(*bad) == 1                                   # NULL weight array
    bad = list(base); bad[2] = nul
    assert f(*bad) == 1 and "layer 1" in moe.moe_last_error_string()
    bad = list(base); bad[12] = P(768)
    assert f(*bad) == 1                                   # scratch aliases y
    bad = list(base); bad[14] = 100
    assert f(*bad) == 1 or f(*bad) == 3                   # never launched: fails before or at the workspace check


def test_noalloc_token_limit_matches_its_documentation():
    """The static scratch of moe_layer_forward_noalloc (32 MiB) holds the
    workspace of up to 314 tokens at the Mixtral-8x7B dimensions, as its
    declaration says; 315 does not fit."""
    cap = 32 << 20
    assert moe.moe_workspace_size(314, 4096, 14336, 8, 2, 0) <= cap
    assert moe.moe_workspace_size(315, 4096, 14336, 8, 2, 0) > cap


def test_test_hooks_validate_their_values():
    """moe_set_gemm_variant takes 0 (automatic) or one of each knob's
    choices; anything else is refused and changes nothing."""
    f = moe.lib.moe_set_gemm_variant
    assert f(4, 0, 0, 0) == 1 and "outside its choices" in moe.moe_last_error_string()
    assert f(-1, 0, 0, 0) == 1
    assert f(0, 64, 0, 0) == 1
    assert f(0, 0, 16, 0) == 1
    assert f(0, 0, 0, 384) == 1
    for args in [(1, 128, 32, 0), (2, 0, 0, 256), (3, 256, 128, 512), (0, 0, 0, 0)]:
        assert f(*args) == 0
    assert moe.lib.moe_set_wait_test(0, 0) == 0
