"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/gka.h declares, and rejects bad arguments with the
documented status codes before any CUDA call."""
import ctypes
import re
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
HEADER = ROOT / "include" / "gka.h"


@pytest.fixture(scope="module")
def lib():
    from test_ridge_regression_b200 import build, gka
    build.build()
    return gka.lib()


def declared_functions():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(gka_[a-z0-9_]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_entry_points():
    names = declared_functions()
    for must in ["gka_forward", "gka_decode_step", "gka_forward_gated", "gka_decode_step_gated",
                 "gka_backward", "gka_backward_workspace_bytes",
                 "gka_forward_workspace_bytes",
                 "gka_forward_workspace_layout", "gka_device_status", "gka_last_cuda_error",
                 "gka_status_string", "gka_version"]:
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(-7, 1):
        assert len(lib.gka_status_string(code)) > 0
    assert lib.gka_version() >= 100


def test_workspace_layout(lib):
    from test_ridge_regression_b200 import gka
    import torch
    B, H, T, D, C = 2, 3, 256, 64, 64
    L = gka.workspace_layout(B, H, T, D, C, torch.float32)
    N = T // C
    assert L.states_offset == 0
    assert L.decay_offset >= 4 * B * H * (N + 1) * 2 * D * D
    assert L.norms_offset >= L.decay_offset + 4 * B * H * N
    assert L.total_bytes >= L.norms_offset + 4 * B * H * T
    for off in (L.states_offset, L.decay_offset, L.norms_offset, L.total_bytes):
        assert off % 256 == 0
    assert gka.workspace_bytes(B, H, T, D, C, torch.float32) == L.total_bytes
    # invalid sizes give 0 bytes
    assert lib.gka_forward_workspace_bytes(1, 1, 100, 64, 64, 0) == 0
    assert lib.gka_forward_workspace_bytes(1, 1, 128, 48, 64, 0) == 0


FAKE = ctypes.c_void_p(1 << 20)       # never dereferenced: every call below fails validation
FAKE_MIS = ctypes.c_void_p((1 << 20) + 4)


def fwd(lib, *, q=FAKE, beta=FAKE, B=1, H=1, T=128, D=64, dt=0, a=0.5, r=4, C=64, ws=FAKE,
        ws_bytes=1 << 40):
    return lib.gka_forward(q, FAKE, FAKE, beta, FAKE, B, H, T, D, dt, a, r, C, None, ws,
                           ws_bytes, None)


def test_forward_argument_errors(lib):
    assert fwd(lib, T=100) == -3                 # T not a multiple of chunk
    assert fwd(lib, D=48) == -2                  # unsupported head dim
    assert fwd(lib, C=96) == -2                  # unsupported chunk
    assert fwd(lib, r=0) == -1
    assert fwd(lib, r=1000) == -2
    assert fwd(lib, a=0.0) == -1
    assert fwd(lib, a=float("nan")) == -1
    assert fwd(lib, a=float("inf")) == -1
    assert fwd(lib, B=-1) == -1
    assert fwd(lib, dt=7) == -1
    assert fwd(lib, q=None) == -1
    assert fwd(lib, q=FAKE_MIS) == -7
    assert fwd(lib, ws_bytes=16) == -4
    assert fwd(lib, B=1000, H=1000) == -2        # more than 65535 heads
    assert fwd(lib, B=0) == 0                    # nothing to do, no launch


def test_decode_argument_errors(lib):
    def dec(state=FAKE, B=2, H=2, D=128, dt=1, a=0.5, r=20):
        return lib.gka_decode_step(state, FAKE, FAKE, FAKE, FAKE, FAKE, B, H, D, dt, a, r, None)
    assert dec(D=96) == -2
    assert dec(r=0) == -1
    assert dec(a=-1.0) == -1
    assert dec(state=None) == -1
    assert dec(state=FAKE_MIS) == -7
    assert dec(B=0) == 0


def test_gated_entry_points_validate_like_the_ungated_ones(lib):
    def fwdg(gate=None, T=128, D=64, r=4):
        return lib.gka_forward_gated(FAKE, FAKE, FAKE, FAKE, gate, FAKE, 1, 1, T, D, 0, 0.5, r,
                                     64, None, FAKE, 1 << 40, None)
    assert fwdg(T=100) == -3
    assert fwdg(D=48) == -2
    assert fwdg(r=0) == -1
    assert fwdg(gate=FAKE_MIS) == -7             # the gate must be 16-byte aligned too

    def decg(gate=None, D=128, r=20):
        return lib.gka_decode_step_gated(FAKE, FAKE, FAKE, FAKE, FAKE, gate, FAKE, 2, 2, D, 1,
                                         0.5, r, None)
    assert decg(D=96) == -2
    assert decg(r=0) == -1
    assert decg(gate=FAKE_MIS) == -7


def test_backward_argument_errors(lib):
    def bwd(gate=None, dgate=None, T=128, D=64, C=32, r=4, q=FAKE, ws_bytes=1 << 40, B=1):
        return lib.gka_backward(q, FAKE, FAKE, FAKE, gate, FAKE, FAKE, FAKE, FAKE, FAKE, dgate,
                                B, 1, T, D, 0, 0.5, r, C, FAKE, ws_bytes, None)
    assert bwd(C=64) == -2                      # the backward takes chunks of 16 or 32
    assert bwd(C=96) == -2
    assert bwd(T=100) == -3
    assert bwd(D=48) == -2
    assert bwd(r=0) == -1
    assert bwd(gate=FAKE) == -1                 # a gate needs its gradient buffer
    assert bwd(dgate=FAKE) == -1                # and a gradient buffer needs a gate
    assert bwd(q=FAKE_MIS) == -7
    assert bwd(gate=FAKE_MIS, dgate=FAKE) == -7
    assert bwd(ws_bytes=16) == -4
    assert bwd(B=0) == 0
    n16 = lib.gka_backward_workspace_bytes(1, 2, 128, 128, 16, 1)
    n32 = lib.gka_backward_workspace_bytes(1, 2, 128, 128, 32, 1)
    assert n16 > n32 > lib.gka_forward_workspace_bytes(1, 2, 128, 128, 64, 1) > 0
    assert lib.gka_backward_workspace_bytes(1, 2, 128, 128, 64, 1) == 0


def test_binding_raises_without_cuda_tensors():
    import torch
    from test_ridge_regression_b200 import gka
    x = torch.zeros(1, 1, 64, 32)
    with pytest.raises(ValueError):
        gka.gka_forward(x, x, x, torch.ones(1, 1, 64), 0.5, 4, 64)


def test_host_forward_plan_and_argument_errors(lib):
    vp = ctypes.c_void_p
    B, H, T, D, C, BF16 = 2, 8, 128, 128, 64, 1
    n_auto = lib.gka_forward_host_workspace_bytes(B, H, T, D, C, BF16, 0)
    n4 = lib.gka_forward_host_workspace_bytes(B, H, T, D, C, BF16, 4)
    assert n_auto > 0 and 0 < n4 < n_auto
    assert lib.gka_forward_host_workspace_bytes(B, H, T, D, C, BF16, -1) == 0
    assert lib.gka_forward_host_workspace_bytes(B, H, 100, D, C, BF16, 0) == 0   # T % C
    fake = vp(1 << 20)
    args = (fake, fake, fake, fake, fake, B, H, T, D, BF16, ctypes.c_float(0.5), 8, C)
    # no workspace, too small a workspace, misaligned workspace, bad a, bad slice
    assert lib.gka_forward_host(*args, None, 0, None, 0, None) == -1
    assert lib.gka_forward_host(*args, None, 0, fake, 256, None) == -4
    assert lib.gka_forward_host(*args, None, 0, vp((1 << 20) + 16), n_auto, None) == -7
    bad_a = args[:10] + (ctypes.c_float(0.0),) + args[11:]
    assert lib.gka_forward_host(*bad_a, None, 0, fake, n_auto, None) == -1
    assert lib.gka_forward_host(*args, None, -3, fake, n_auto, None) == -1
