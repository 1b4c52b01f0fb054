"""C-ABI host logic without a GPU: the library loads, exports every symbol the
header declares, and rejects invalid arguments before touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import efficient_vision_attention_b200 as eva
from efficient_vision_attention_b200 import binding
from efficient_vision_attention_b200.build import LIB, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "agent_attn.h")

A16 = 1 << 20          # a fake, 16-byte aligned address: never dereferenced
ODD = A16 + 8          # 8-byte aligned only


@pytest.fixture(scope="module", autouse=True)
def built():
    build()


def header_functions():
    text = open(HEADER).read()
    return re.findall(r"^AA_API\s+[\w\s\*]+?\b(agent_attn_\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_boundary():
    names = set(header_functions())
    for n in ["agent_attn_forward", "agent_attn_forward_agents", "agent_attn_workspace_bytes",
              "agent_attn_forward_ws", "agent_attn_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\sT\s(\w+)$", out, flags=re.M))
    declared = set(header_functions())
    assert declared <= exported, declared - exported
    # nothing but the declared C ABI leaks out of the library
    ours = {s for s in exported if s.startswith("agent_attn")}
    assert ours == declared
    # and the binding wraps exactly those names
    assert set(binding.exported_symbols()) == declared


def test_header_compiles_as_c():
    src = '#include "agent_attn.h"\nint main(void){return (int)AA_OK;}\n'
    r = subprocess.run(["gcc", "-x", "c", "-std=c99", "-fsyntax-only", "-I",
                        os.path.join(ROOT, "include"), "-"], input=src, text=True,
                       capture_output=True)
    assert r.returncode == 0, r.stderr


def test_status_strings():
    for code in range(9):
        s = eva.agent_attn_status_string(code)
        assert s and binding.STATUS_NAMES[code] in s
    assert "unknown" in eva.agent_attn_status_string(99)
    assert re.match(r"\d+\.\d+\.\d+", binding.agent_attn_version())


def fwd(**kw):
    args = dict(q=A16, k=A16, v=A16, agents_or_null=None, out=A16, B=2, H=3, N=196, d=64,
                grid_h=14, grid_w=14, pool_h=7, pool_w=7, scale=0.125, dtype=eva.AA_BF16,
                stream=0, check=False)
    args.update(kw)
    return eva.agent_attn_forward(**args)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(k=None), 1), (dict(v=None), 1), (dict(out=None), 1),
    (dict(q=ODD), 4), (dict(out=ODD), 4), (dict(agents_or_null=ODD), 4),
    (dict(N=195), 2), (dict(grid_h=13), 2), (dict(pool_h=15), 2), (dict(pool_w=0), 2),
    (dict(B=0), 2), (dict(H=-1), 2), (dict(N=0, grid_h=0, grid_w=0), 2),
    (dict(d=40 + 4), 3), (dict(d=136), 3), (dict(d=0), 3), (dict(dtype=7), 3),
    (dict(grid_h=20, grid_w=20, N=400, pool_h=17, pool_w=16), 3),   # 272 agents > 256
    (dict(scale=0.0), 7), (dict(scale=float("nan")), 7), (dict(scale=float("inf")), 7),
    (dict(scale=-1.0), 7),
])
def test_forward_rejects_invalid_arguments(kw, status):
    assert fwd(**kw) == status


def test_forward_agents_and_stage_validation():
    base = dict(q=A16, k=A16, v=A16, agents=A16, n_agents=49, agents_batch_stride=0, out=A16,
                B=1, H=2, N=100, d=32, scale=0.2, dtype=eva.AA_BF16, stream=0, check=False)
    f = eva.agent_attn_forward_agents
    assert f(**{**base, "agents": None}) == 1
    assert f(**{**base, "agents": ODD}) == 4
    assert f(**{**base, "agents_batch_stride": 12}) == 4
    assert f(**{**base, "agents_batch_stride": -8}) == 4
    assert f(**{**base, "n_agents": 0}) == 3
    assert f(**{**base, "n_agents": 257}) == 3
    assert eva.agent_attn_stage_pool(A16, None, None, 1, 1, 64, 32, 8, 8, 2, 2, eva.AA_BF16, 0,
                                     check=False) == 1
    assert eva.agent_attn_stage_pool(A16, A16, None, 1, 1, 64, 32, 8, 8, 9, 2, eva.AA_FP32, 0,
                                     check=False) == 2
    assert eva.agent_attn_stage_aggregate(A16, 0, A16, A16, None, None, 1, 1, 64, 32, 4, 0.1,
                                          eva.AA_FP32, 0, check=False) == 1
    assert eva.agent_attn_stage_broadcast(A16, A16, 0, A16, A16, 1, 1, 64, 32, 4, 0.0,
                                          eva.AA_FP32, 0, check=False) == 7


def test_workspace_validation():
    ws = dict(q=A16, k=A16, v=A16, agents_or_null=None, out=A16, B=1, H=1, N=64, d=32, grid_h=8,
              grid_w=8, pool_h=2, pool_w=2, scale=0.1, dtype=eva.AA_FP32, stream=0, check=False)
    assert eva.agent_attn_forward_ws(**ws, workspace=None, ws_bytes=1 << 20) in (1, 6)
    assert eva.agent_attn_workspace_bytes(1, 1, 64, 33, 4, eva.AA_FP32) == 0
    assert eva.agent_attn_workspace_bytes(1, 1, 64, 32, 0, eva.AA_FP32) == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_valid_call_without_a_device_reports_cuda_error():
    """With no usable device the first CUDA call fails; the library returns
    AA_ERR_CUDA and keeps the CUDA error text (a host-side injected failure)."""
    assert fwd() == 6
    assert "cuda" in eva.agent_attn_status_string(6).lower()
    assert eva.agent_attn_workspace_bytes(1, 1, 64, 32, 4, eva.AA_FP32) == 0


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setenv("AGENT_ATTN_LIB", str(tmp_path / "nope.so"))
    with pytest.raises(binding.AgentAttnError, match="missing"):
        binding.load_library()
    monkeypatch.setattr(binding, "_lib", None)


def test_dwc_validation():
    base = dict(v=A16, w=A16, bias_or_null=None, out=A16, B=1, H=2, grid_h=8, grid_w=8, d=32,
                dtype=eva.AA_BF16, accumulate=True, stream=0, check=False)
    f = eva.agent_attn_dwc
    assert f(**{**base, "v": None}) == 1
    assert f(**{**base, "w": None}) == 1
    assert f(**{**base, "out": ODD}) == 4
    assert f(**{**base, "d": 36}) == 3
    assert f(**{**base, "d": 136}) == 3
    assert f(**{**base, "dtype": 5}) == 3
    assert f(**{**base, "grid_w": 0}) == 2
    # a slice of 2^31 8-channel groups or more is refused before any launch
    assert f(**{**base, "grid_h": 1 << 16, "grid_w": 1 << 13, "d": 32}) == 2
    g = eva.agent_attn_forward_dwc
    full = dict(q=A16, k=A16, v=A16, agents_or_null=None, dwc_w=A16, dwc_bias_or_null=None,
                out=A16, B=1, H=1, N=64, d=32, grid_h=8, grid_w=8, pool_h=2, pool_w=2, scale=0.1,
                dtype=eva.AA_BF16, stream=0, check=False)
    assert g(**{**full, "dwc_w": None}) == 1
    assert g(**{**full, "N": 63}) == 2
    assert g(**{**full, "pool_h": 9}) == 2


def test_bias_validation():
    base = dict(q=A16, k=A16, v=A16, agents_or_null=None, b1=(A16, None, None), b2=None, out=A16,
                B=1, H=1, N=64, d=32, grid_h=8, grid_w=8, pool_h=2, pool_w=2, scale=0.1,
                dtype=eva.AA_BF16, stream=0, check=False)
    f = eva.agent_attn_forward_bias
    assert f(**{**base, "b1": (A16 + 2, None, None)}) == 4
    assert f(**{**base, "b2": (None, None, A16 + 1)}) == 4
    assert f(**{**base, "N": 65}) == 2
    assert f(**{**base, "q": None}) == 1
    assert f(**{**base, "scale": -1.0}) == 7


def test_backward_validation():
    base = dict(q=A16, k=A16, v=A16, agents_or_null=None, dout=A16, dq=A16, dk=A16, dv=A16,
                dagents_or_null=None, B=1, H=1, N=64, d=32, grid_h=8, grid_w=8, pool_h=2,
                pool_w=2, scale=0.1, dtype=eva.AA_BF16, stream=0, check=False)
    f = eva.agent_attn_backward
    assert f(**{**base, "dout": None}) == 1
    assert f(**{**base, "dk": None}) == 1
    assert f(**{**base, "dv": ODD}) == 4
    assert f(**{**base, "dagents_or_null": A16 + 2}) == 4
    assert f(**{**base, "N": 60}) == 2
    assert f(**{**base, "B": 70000, "H": 1}) == 2
