"""ctypes binding of ``libagentattn.so`` (declared in ``include/agent_attn.h``).

Argument marshalling only: every function forwards to the C entry point of
the same name.  Tensor arguments may be torch tensors (their data pointer is
passed) or plain integer addresses; ``stream`` may be a ``torch.cuda.Stream``,
an integer handle or None (torch's current stream on the current device).
A non-zero status raises :class:`AgentAttnError` unless ``check=False``, in
which case the status code is returned.  There is no fallback: if the library
is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os

AA_FP32 = 0
AA_BF16 = 1

STATUS_NAMES = {0: "AA_OK", 1: "AA_ERR_NULL", 2: "AA_ERR_SHAPE", 3: "AA_ERR_UNSUPPORTED",
                4: "AA_ERR_ALIGN", 5: "AA_ERR_WORKSPACE", 6: "AA_ERR_CUDA", 7: "AA_ERR_VALUE",
                8: "AA_ERR_TIMEOUT"}

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libagentattn.so"
_lib = None

_vp = ctypes.c_void_p
_i = ctypes.c_int
_ll = ctypes.c_longlong
_f = ctypes.c_float
_sz = ctypes.c_size_t

_SIGNATURES = {
    "agent_attn_forward": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f, _i, _vp]),
    "agent_attn_forward_ws": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f, _i,
                                   _vp, _sz, _vp]),
    "agent_attn_forward_agents": (_i, [_vp, _vp, _vp, _vp, _i, _ll, _vp, _i, _i, _i, _i, _f, _i,
                                       _vp]),
    "agent_attn_workspace_bytes": (_sz, [_i, _i, _i, _i, _i, _i]),
    "agent_attn_forward_host": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f,
                                     _i, _vp]),
    "agent_attn_stage_pool": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "agent_attn_stage_aggregate": (_i, [_vp, _ll, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i,
                                        _vp]),
    "agent_attn_stage_broadcast": (_i, [_vp, _vp, _ll, _vp, _vp, _i, _i, _i, _i, _i, _f, _i,
                                        _vp]),
    "agent_attn_status_string": (ctypes.c_char_p, [_i]),
    "agent_attn_version": (ctypes.c_char_p, []),
    "agent_attn_check_device_error": (_i, []),
    "agent_attn_stage_aggregate_static": (_i, [_vp, _ll, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                                               _f, _i, _vp]),
    "agent_attn_forward_bias": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i,
                                     _i, _i, _i, _i, _i, _i, _f, _i, _vp]),
    "agent_attn_backward": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                                 _i, _i, _i, _f, _i, _vp]),
    "agent_attn_dwc": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "agent_attn_forward_dwc": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                    _i, _f, _i, _vp]),
    "agent_attn_selftest_exp2": (_i, [_vp, _vp, _vp, _i, _vp]),
}

# Size of the library's fixed scratch array (AA_STATIC_SCRATCH_BYTES in the header).
AA_STATIC_SCRATCH_BYTES = 16 << 20


class AgentAttnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def library_path() -> str:
    return os.environ.get("AGENT_ATTN_LIB", os.path.join(_PKG, _LIB_NAME))


def load_library():
    """Loads the CUDA library; raises AgentAttnError if it is not built."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise AgentAttnError(-1, f"{path} is missing: build it with "
                                     "`python -m efficient_vision_attention_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def exported_symbols() -> list[str]:
    return list(_SIGNATURES)


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _finish(status: int, check: bool):
    if status != 0 and check:
        raise AgentAttnError(status, agent_attn_status_string(status))
    return status


def agent_attn_status_string(status: int) -> str:
    return load_library().agent_attn_status_string(int(status)).decode()


def agent_attn_version() -> str:
    return load_library().agent_attn_version().decode()


def agent_attn_forward(q, k, v, agents_or_null, out, B, H, N, d, grid_h, grid_w, pool_h, pool_w,
                       scale, dtype, stream=None, check=True):
    st = load_library().agent_attn_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(agents_or_null),
                                           _ptr(out), B, H, N, d, grid_h, grid_w, pool_h, pool_w,
                                           scale, dtype, _stream(stream))
    return _finish(st, check)


def agent_attn_forward_ws(q, k, v, agents_or_null, out, B, H, N, d, grid_h, grid_w, pool_h,
                          pool_w, scale, dtype, workspace, ws_bytes, stream=None, check=True):
    st = load_library().agent_attn_forward_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(agents_or_null),
                                              _ptr(out), B, H, N, d, grid_h, grid_w, pool_h,
                                              pool_w, scale, dtype, _ptr(workspace), ws_bytes,
                                              _stream(stream))
    return _finish(st, check)


def agent_attn_forward_agents(q, k, v, agents, n_agents, agents_batch_stride, out, B, H, N, d,
                              scale, dtype, stream=None, check=True):
    st = load_library().agent_attn_forward_agents(_ptr(q), _ptr(k), _ptr(v), _ptr(agents),
                                                  n_agents, agents_batch_stride, _ptr(out), B, H,
                                                  N, d, scale, dtype, _stream(stream))
    return _finish(st, check)


def agent_attn_workspace_bytes(B, H, N, d, n_agents, dtype) -> int:
    return int(load_library().agent_attn_workspace_bytes(B, H, N, d, n_agents, dtype))


def agent_attn_forward_host(q_host, k_host, v_host, agents_host_or_null, out_host, B, H, N, d,
                            grid_h, grid_w, pool_h, pool_w, scale, dtype, stream=None,
                            check=True):
    st = load_library().agent_attn_forward_host(_ptr(q_host), _ptr(k_host), _ptr(v_host),
                                                _ptr(agents_host_or_null), _ptr(out_host), B, H,
                                                N, d, grid_h, grid_w, pool_h, pool_w, scale,
                                                dtype, _stream(stream))
    return _finish(st, check)


def agent_attn_stage_pool(q, agents_f32, agents_lowp, B, H, N, d, grid_h, grid_w, pool_h, pool_w,
                          dtype, stream=None, check=True):
    st = load_library().agent_attn_stage_pool(_ptr(q), _ptr(agents_f32), _ptr(agents_lowp), B, H,
                                              N, d, grid_h, grid_w, pool_h, pool_w, dtype,
                                              _stream(stream))
    return _finish(st, check)


def agent_attn_stage_aggregate(agents, agents_batch_stride, k, v, va_f32, va_lowp, B, H, N, d,
                               n_agents, scale, dtype, stream=None, check=True):
    st = load_library().agent_attn_stage_aggregate(_ptr(agents), agents_batch_stride, _ptr(k),
                                                   _ptr(v), _ptr(va_f32), _ptr(va_lowp), B, H, N,
                                                   d, n_agents, scale, dtype, _stream(stream))
    return _finish(st, check)


def agent_attn_stage_broadcast(q, agents, agents_batch_stride, va, out, B, H, N, d, n_agents,
                               scale, dtype, stream=None, check=True):
    st = load_library().agent_attn_stage_broadcast(_ptr(q), _ptr(agents), agents_batch_stride,
                                                   _ptr(va), _ptr(out), B, H, N, d, n_agents,
                                                   scale, dtype, _stream(stream))
    return _finish(st, check)


def agent_attn_check_device_error(check=True):
    return _finish(load_library().agent_attn_check_device_error(), check)


def agent_attn_stage_aggregate_static(agents, agents_batch_stride, k, v, va_f32, va_lowp, B, H,
                                      N, d, n_agents, scale, dtype, stream=None, check=True):
    """Aggregation stage that allocates nothing: the split partials live in a
    fixed array inside the library.  For callers that may not allocate device
    memory (a plugin in a framework that owns the device memory, a loop that
    forbids allocation after start-up).  Make the first call on a device
    before any stream capture; calls that overlap on the GPU share the array
    and race, so serialise them."""
    st = load_library().agent_attn_stage_aggregate_static(
        _ptr(agents), agents_batch_stride, _ptr(k), _ptr(v), _ptr(va_f32), _ptr(va_lowp), B, H, N,
        d, n_agents, scale, dtype, _stream(stream))
    return _finish(st, check)


def agent_attn_dwc(v, w, bias_or_null, out, B, H, grid_h, grid_w, d, dtype, accumulate=False,
                   stream=None, check=True):
    """out (+)= depth-wise 3x3 convolution of v over its token grid; w is
    [H, d, 3, 3] fp32, bias [H, d] fp32 or None."""
    st = load_library().agent_attn_dwc(_ptr(v), _ptr(w), _ptr(bias_or_null), _ptr(out), B, H,
                                       grid_h, grid_w, d, dtype, 1 if accumulate else 0,
                                       _stream(stream))
    return _finish(st, check)


def agent_attn_forward_dwc(q, k, v, agents_or_null, dwc_w, dwc_bias_or_null, out, B, H, N, d,
                           grid_h, grid_w, pool_h, pool_w, scale, dtype, stream=None, check=True):
    """The full module output: the forward pass plus the depth-wise convolution of v."""
    st = load_library().agent_attn_forward_dwc(_ptr(q), _ptr(k), _ptr(v), _ptr(agents_or_null),
                                               _ptr(dwc_w), _ptr(dwc_bias_or_null), _ptr(out), B,
                                               H, N, d, grid_h, grid_w, pool_h, pool_w, scale,
                                               dtype, _stream(stream))
    return _finish(st, check)


def agent_attn_forward_bias(q, k, v, agents_or_null, b1, b2, out, B, H, N, d, grid_h, grid_w,
                            pool_h, pool_w, scale, dtype, stream=None, check=True):
    """Forward pass with agent bias.  b1, b2: (row, col, block) triples of fp32
    device tensors [H, k, grid_h], [H, k, grid_w], [H, k, pool_h*pool_w]
    (entries may be None), or None for no bias on that softmax."""
    r1, c1, k1 = b1 if b1 is not None else (None, None, None)
    r2, c2, k2 = b2 if b2 is not None else (None, None, None)
    st = load_library().agent_attn_forward_bias(
        _ptr(q), _ptr(k), _ptr(v), _ptr(agents_or_null), _ptr(r1), _ptr(c1), _ptr(k1), _ptr(r2),
        _ptr(c2), _ptr(k2), _ptr(out), B, H, N, d, grid_h, grid_w, pool_h, pool_w, scale, dtype,
        _stream(stream))
    return _finish(st, check)


def agent_attn_backward(q, k, v, agents_or_null, dout, dq, dk, dv, dagents_or_null, B, H, N, d,
                        grid_h, grid_w, pool_h, pool_w, scale, dtype, stream=None, check=True):
    """Gradients dq, dk, dv (and the agents' own gradient, fp32 [B, H, k, d],
    when dagents_or_null is given) of the forward pass for dout."""
    st = load_library().agent_attn_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(agents_or_null), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
        _ptr(dagents_or_null), B, H, N, d, grid_h, grid_w, pool_h, pool_w, scale, dtype,
        _stream(stream))
    return _finish(st, check)


def agent_attn_selftest_exp2(x, y_fma, y_ref, n, stream=None, check=True):
    return _finish(load_library().agent_attn_selftest_exp2(_ptr(x), _ptr(y_fma), _ptr(y_ref),
                                                           int(n), _stream(stream)), check)
