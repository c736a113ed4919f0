"""CPU checks of the C-ABI library: it loads without a GPU, exports every
function include/rglru.h declares, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import pytest

from gated_linear_recurrence_rglru_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[a-z_]+\s*\*?\s*(rglru_[a-z0-9_]+)\s*\(",
                                src, flags=re.M)
    return names


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("rglru_fwd", "rglru_decode_step", "rglru_fwd_workspace_bytes"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(_abi.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert set(_abi.EXPORTED) <= set(declared_functions())


def test_status_strings_and_version():
    assert _abi.status_str(0) == "ok"
    assert "timed out" in _abi.status_str(4)
    assert _abi.status_str(99) == "unknown status"
    assert _abi.version() >= 100


def test_workspace_bytes():
    lib = _abi.LIB
    assert lib.rglru_fwd_workspace_bytes(8, 2048, 1024, 16, 1) >= 256
    assert lib.rglru_fwd_workspace_bytes(0, 2048, 1024, 16, 1) == 0
    assert lib.rglru_fwd_workspace_bytes(8, 2048, 1000, 16, 1) == 0      # D % H != 0
    assert lib.rglru_fwd_workspace_bytes(8, 2048, 1024, 16, 7) == 0      # bad io
    # more segments (smaller B*H) never needs less than a single long segment
    assert lib.rglru_fwd_workspace_bytes(1, 131072, 4096, 16, 1) > 0


FAKE = 1 << 20  # 16-byte aligned non-null stand-in; never dereferenced: the checks fail first


def fwd_call(**over):
    a = dict(x=FAKE, conv_w=FAKE, W_a=FAKE, b_a=FAKE, W_x=FAKE, b_x=FAKE, Lambda=FAKE, h0=None,
             csi=None, y=FAKE * 64, h_T=None, cso=None, B=2, T=16, D=64, H=2, io=1,
             ws=FAKE * 128, ws_bytes=1 << 30, dev_status=None, stream=None, algo=0)
    a.update(over)
    return _abi.LIB.rglru_fwd_algo(a["x"], a["conv_w"], a["W_a"], a["b_a"], a["W_x"], a["b_x"],
                                   a["Lambda"], a["h0"], a["csi"], a["y"], a["h_T"], a["cso"],
                                   a["B"], a["T"], a["D"], a["H"], a["io"], a["ws"],
                                   a["ws_bytes"], a["dev_status"], a["stream"], a["algo"])


@pytest.mark.parametrize("over,code", [
    (dict(B=0), 1), (dict(T=0), 1), (dict(H=0), 1), (dict(D=60, H=2), 1), (dict(D=63, H=1), 1),
    (dict(io=3), 1), (dict(x=None), 1), (dict(Lambda=None), 1), (dict(y=None), 1),
    (dict(x=FAKE + 4), 1), (dict(h0=FAKE + 8), 1), (dict(y=FAKE), 1),          # y aliases x
    (dict(D=2048, H=1), 2), (dict(algo=9), 1),
    (dict(B=64, T=4096, ws=None), 5), (dict(B=64, T=4096, ws_bytes=16), 5),
])
def test_fwd_rejects_bad_arguments(over, code):
    assert fwd_call(**over) == code


def test_decode_rejects_bad_arguments():
    L = _abi.LIB
    args = [FAKE, FAKE * 2, 0, FAKE * 4, FAKE * 8, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 64, 2, 1,
            None, 0]
    bad = list(args); bad[2] = -1
    assert L.rglru_decode_step_algo(*bad) == 1                 # pos < 0
    bad = list(args); bad[4] = FAKE                            # y_t aliases x_t
    assert L.rglru_decode_step_algo(*bad) == 1
    bad = list(args); bad[13] = 3                              # D % H
    assert L.rglru_decode_step_algo(*bad) == 1
    bad = list(args); bad[3] = None
    assert L.rglru_decode_step_algo(*bad) == 1


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 4, 8)
    with pytest.raises((TypeError, RuntimeError)):
        _abi.rglru_fwd(x, torch.zeros(4, 8), torch.zeros(1, 8, 8), torch.zeros(8),
                       torch.zeros(1, 8, 8), torch.zeros(8), torch.zeros(8))


def test_options_struct_matches_header():
    """The ctypes mirror of rglru_fwd_options has the header's fields in order."""
    from gated_linear_recurrence_rglru_b200._abi import FwdOptions
    hdr = open(os.path.join(ROOT, "include", "rglru.h")).read()
    body = re.search(r"typedef struct \{([^}]*)\} rglru_fwd_options;", hdr).group(1)
    names = re.findall(r"(\w+)\s*;", body)
    assert names == [f[0] for f in FwdOptions._fields_]


def test_bwd_refuses_bad_arguments_before_launch():
    """rglru_bwd (28 arguments) checks shapes and pointers on the host."""
    L = _abi.LIB
    null = [None] * 20
    # null required pointers
    assert L.rglru_bwd(*null, 2, 8, 64, 2, 0, None, 0, None) == 1
    # bad shapes: D not a multiple of H, bad io
    assert L.rglru_bwd(*null, 2, 8, 65, 2, 0, None, 0, None) == 1
    assert L.rglru_bwd(*null, 2, 8, 64, 2, 7, None, 0, None) == 1
    assert L.rglru_bwd_workspace_bytes(2, 8, 64, 2, 0) > 0
    assert L.rglru_bwd_workspace_bytes(2, 8, 65, 2, 0) == 0
    assert L.rglru_bwd_launches(2, 8, 64, 2, 1) == 5


def test_block_refuses_bad_arguments_before_launch():
    """rglru_block_fwd (25 arguments) checks shapes, pointers, overlaps and the
    workspace on the host, before any CUDA call."""
    L = _abi.LIB
    B, T, Dm, D, H, io = 2, 8, 64, 64, 2, 0
    # x, W_in, W_gate, W_out, conv_w, W_a, b_a, W_x, b_x, Lambda, h0, conv_state_in, out, h_T,
    # conv_state_out: distinct 16-byte aligned stand-ins 1 MiB apart (never dereferenced)
    ptrs = [FAKE * (k + 1) for k in range(15)]
    ptrs[10] = ptrs[11] = ptrs[13] = ptrs[14] = None          # optional ones absent
    ws_need = L.rglru_block_fwd_workspace_bytes(B, T, Dm, D, H, io)
    assert ws_need > 0
    assert L.rglru_block_fwd_workspace_bytes(B, T, 12, D, H, io) == 0      # Dm % 8
    assert L.rglru_block_fwd_workspace_bytes(B, T, Dm, 65, H, io) == 0     # D % H

    def call(p=ptrs, dims=(B, T, Dm, D, H, io), ws=None, ws_bytes=0):
        return L.rglru_block_fwd(*p, *dims, ws, ws_bytes, None, None)

    assert call(p=[None] * 15) == 1                              # null required pointers
    assert call(dims=(B, T, 12, D, H, io)) == 1                  # Dm not a multiple of 8
    assert call(dims=(B, T, Dm, D, H, 7)) == 1                   # bad io
    bad = list(ptrs); bad[12] = ptrs[0]                          # out aliases x
    assert call(p=bad) == 1
    assert call() == 5                                           # no workspace
    assert call(ws=FAKE * 64, ws_bytes=ws_need - 16) == 5        # workspace too small
