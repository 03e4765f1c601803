"""ctypes binding of libla2.so (C ABI in ``include/la2.h``).

Argument marshalling only: every step of the computation runs in the
library's CUDA kernels. The raw functions keep the C names and argument order
and return the C status code. ``forward`` / ``backward`` below take torch
tensors, allocate outputs and the workspace with torch (PyTorch is only the
allocator and the stream provider here) and raise ``La2Error`` on a non-zero
status. Importing this module fails loudly when the library is missing.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libla2.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libla2.so not found at {LIB_PATH}; build it with "
        "`python -m linear_attention_la2_b200.build` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

LA2_OK = 0
LA2_ERR_INVALID_ARG = 1
LA2_ERR_UNSUPPORTED = 2
LA2_ERR_WORKSPACE = 3
LA2_ERR_CUDA = 4
LA2_ERR_TIMEOUT = 5
LA2_F32 = 0
LA2_BF16 = 1

_i64 = ctypes.c_int64
_int = ctypes.c_int
_vp = ctypes.c_void_p
_sz = ctypes.c_size_t

_SIGS = {
    "la2_workspace_size": (_sz, [_i64, _i64, _i64, _i64, _i64, _int, _int, _int, _int]),
    "la2_forward": (_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _int, _int, _int,
                           _vp, _sz, _vp]),
    "la2_backward": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _int,
                            _int, _int, _vp, _sz, _vp]),
    "la2_workspace_size_gqa": (_sz, [_i64, _i64, _i64, _i64, _i64, _i64, _int, _int, _int, _int]),
    "la2_forward_gqa": (_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64, _int, _int,
                               _int, _vp, _sz, _vp]),
    "la2_backward_gqa": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64,
                                _i64, _int, _int, _int, _vp, _sz, _vp]),
    "la2_workspace_size_sp": (_sz, [_i64, _i64, _i64, _i64, _i64, _int, _int, _int]),
    "la2_forward_sp": (_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64, _int,
                              _int, _vp, _sz, _vp]),
    "la2_backward_sp": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _i64, _i64, _i64,
                               _i64, _i64, _i64, _int, _int, _vp, _sz, _vp]),
    "la2_workspace_size_decay": (_sz, [_i64, _i64, _i64, _i64, _i64, _int, _int, _int]),
    "la2_forward_decay": (_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _int, _int,
                                 _vp, _sz, _vp]),
    "la2_backward_decay": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                  _i64, _int, _int, _vp, _sz, _vp]),
    "la2_check": (_int, [_vp]),
    "la2_status_string": (ctypes.c_char_p, [_int]),
    "la2_set_chunk_len": (_int, [_i64]),
    "la2_plan_ranges": (_i64, [_i64, _i64, _i64, _i64, _i64, _int, _int, _int, _int,
                               ctypes.POINTER(_i64), _i64]),
    "la2_set_spin_limit": (_int, [_i64]),
    "la2_profile_enable": (_int, [_int]),
    "la2_profile_num_kernels": (_int, []),
    "la2_profile_kernel_name": (ctypes.c_char_p, [_int]),
    "la2_profile_collect": (_int, [_int, ctypes.POINTER(_i64), ctypes.POINTER(ctypes.c_double)]),
    "la2_version": (_int, []),
    "la2_forward_noalloc": (_int, [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _int, _int,
                                   _int, _vp]),
    "la2_kv_state_workspace_size": (_sz, [_i64, _i64, _i64, _i64, _i64, _int]),
    "la2_kv_state": (_int, [_vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _int, _vp, _sz, _vp]),
    "la2_decode_step": (_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _int, _vp]),
}

EXPORTED = tuple(_SIGS)

for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

# Raw C entry points, same names and argument order as include/la2.h.
la2_workspace_size = _lib.la2_workspace_size
la2_forward = _lib.la2_forward
la2_backward = _lib.la2_backward
la2_check = _lib.la2_check
la2_workspace_size_gqa = _lib.la2_workspace_size_gqa
la2_forward_gqa = _lib.la2_forward_gqa
la2_backward_gqa = _lib.la2_backward_gqa
la2_workspace_size_sp = _lib.la2_workspace_size_sp
la2_forward_sp = _lib.la2_forward_sp
la2_backward_sp = _lib.la2_backward_sp
la2_workspace_size_decay = _lib.la2_workspace_size_decay
la2_forward_decay = _lib.la2_forward_decay
la2_backward_decay = _lib.la2_backward_decay
la2_set_chunk_len = _lib.la2_set_chunk_len
la2_plan_ranges = _lib.la2_plan_ranges
la2_set_spin_limit = _lib.la2_set_spin_limit
la2_profile_enable = _lib.la2_profile_enable
la2_profile_num_kernels = _lib.la2_profile_num_kernels
la2_version = _lib.la2_version
la2_forward_noalloc = _lib.la2_forward_noalloc
la2_kv_state_workspace_size = _lib.la2_kv_state_workspace_size
la2_kv_state = _lib.la2_kv_state
la2_decode_step = _lib.la2_decode_step
NOALLOC_SCRATCH_BYTES = 32 << 20


def plan_ranges(B, H, N, d, dv, causal, block, dtype_code, is_backward=False):
    """Range starts (in blocks of the flattened B*H*ceil(N/block) list) the
    library will use for these arguments."""
    R = la2_plan_ranges(B, H, N, d, dv, int(causal), block, dtype_code, int(is_backward), None, 0)
    if R < 0:
        raise La2Error(LA2_ERR_INVALID_ARG)
    buf = (_i64 * (R + 1))()
    la2_plan_ranges(B, H, N, d, dv, int(causal), block, dtype_code, int(is_backward), buf, R + 1)
    return list(buf)


def la2_status_string(code: int) -> str:
    return _lib.la2_status_string(code).decode()


def la2_profile_kernel_name(kernel: int) -> str:
    s = _lib.la2_profile_kernel_name(kernel)
    return s.decode() if s else ""


def la2_profile_collect(kernel: int):
    n = _i64(0)
    ms = ctypes.c_double(0.0)
    st = _lib.la2_profile_collect(kernel, ctypes.byref(n), ctypes.byref(ms))
    _raise(st)
    return int(n.value), float(ms.value)


class La2Error(RuntimeError):
    def __init__(self, code: int):
        super().__init__(la2_status_string(code))
        self.code = code


def _raise(code: int):
    if code != LA2_OK:
        raise La2Error(code)


# ------------------------------------------------------------ torch helpers


def _dtype_code(t):
    import torch

    if t.dtype == torch.bfloat16:
        return LA2_BF16
    if t.dtype == torch.float32:
        return LA2_F32
    raise La2Error(LA2_ERR_UNSUPPORTED)


def _stream_handle(stream):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return _vp(stream.cuda_stream)


def _ptr(t):
    return _vp(t.data_ptr()) if t is not None and t.numel() > 0 else _vp(0)


def workspace_bytes(B, H, N, d, dv, causal, block, dtype_code, is_backward) -> int:
    n = la2_workspace_size(B, H, N, d, dv, int(causal), block, dtype_code, int(is_backward))
    if n == ctypes.c_size_t(-1).value:
        raise La2Error(LA2_ERR_INVALID_ARG)
    return int(n)


def _workspace(nbytes, device, stream):
    """Scratch for one call, allocated on the stream the kernels run on, so the
    caching allocator cannot hand it to other work while they still use it."""
    import torch

    if nbytes == 0:
        return None
    if stream is None:
        return torch.empty(nbytes, dtype=torch.uint8, device=device)
    with torch.cuda.stream(stream):
        return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _check_inputs(*ts):
    for t in ts:
        if not t.is_cuda:
            raise La2Error(LA2_ERR_INVALID_ARG)
        if not t.is_contiguous():
            raise La2Error(LA2_ERR_INVALID_ARG)


def _check_like(ref, shape, dtype, *ts):
    """Every tensor in ``ts`` must have ``shape``, ``dtype`` and ref's device:
    the library sizes every tensor map and loop from q's shape, so a shorter
    k, v, dO or output would be read or written past its end."""
    for t in ts:
        if tuple(t.shape) != tuple(shape) or t.dtype != dtype or t.device != ref.device:
            raise La2Error(LA2_ERR_INVALID_ARG)


def _check_workspace(ws, need, device):
    import torch

    if ws is None:
        if need:
            raise La2Error(LA2_ERR_WORKSPACE)
        return
    if not ws.is_cuda or ws.device != device or not ws.is_contiguous() or ws.dtype != torch.uint8:
        raise La2Error(LA2_ERR_INVALID_ARG)


def _kv_heads(q, k, v):
    """K/V head count of a call: k, v [B,Hkv,N,.] with Hkv dividing q's H."""
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise La2Error(LA2_ERR_INVALID_ARG)
    H, Hkv = q.shape[1], k.shape[1]
    if (H > 0 and (Hkv < 1 or H % Hkv)) or (H == 0 and Hkv != 0):
        raise La2Error(LA2_ERR_INVALID_ARG)
    return Hkv


def workspace_bytes_gqa(B, H, Hkv, N, d, dv, causal, block, dtype_code, is_backward) -> int:
    n = la2_workspace_size_gqa(B, H, Hkv, N, d, dv, int(causal), block, dtype_code, int(is_backward))
    if n == ctypes.c_size_t(-1).value:
        raise La2Error(LA2_ERR_INVALID_ARG)
    return int(n)


def forward(q, k, v, causal: bool = True, block: int = 64, out=None, workspace=None, stream=None):
    """O = ((Q K^T) ⊙ M) V for [B,H,N,d] CUDA tensors; returns O. k and v may
    hold fewer heads (grouped K/V heads: query head h reads K/V head
    h // (H // Hkv))."""
    import torch

    _check_inputs(q, k, v)
    Hkv = _kv_heads(q, k, v)
    B, H, N, d = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    _check_like(q, (B, Hkv, N, d), q.dtype, k)
    _check_like(q, (B, Hkv, N, dv), q.dtype, v)
    if out is None:
        out = torch.empty((B, H, N, dv), dtype=q.dtype, device=q.device)
    _check_inputs(out)
    _check_like(q, (B, H, N, dv), q.dtype, out)
    need = workspace_bytes_gqa(B, H, Hkv, N, d, dv, causal, block, dt, False)
    ws = workspace if workspace is not None else _workspace(need, q.device, stream)
    _check_workspace(ws, need, q.device)
    _raise(la2_forward_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, Hkv, N, d, dv, int(causal),
                           block, dt, _ptr(ws), ws.numel() if ws is not None else 0,
                           _stream_handle(stream)))
    return out


def backward(q, k, v, do, causal: bool = True, block: int = 64, outs=None, workspace=None,
             stream=None):
    """Gradients (dQ, dK, dV) of <dO, O> for the same op; returns a tuple. With
    grouped K/V heads dK and dV are the sums over each group's query heads."""
    import torch

    _check_inputs(q, k, v, do)
    Hkv = _kv_heads(q, k, v)
    B, H, N, d = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    _check_like(q, (B, Hkv, N, d), q.dtype, k)
    _check_like(q, (B, Hkv, N, dv), q.dtype, v)
    _check_like(q, (B, H, N, dv), q.dtype, do)
    if outs is None:
        outs = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    dq, dk, dvv = outs
    _check_inputs(dq, dk, dvv)
    _check_like(q, q.shape, q.dtype, dq)
    _check_like(q, (B, Hkv, N, d), q.dtype, dk)
    _check_like(q, (B, Hkv, N, dv), q.dtype, dvv)
    need = workspace_bytes_gqa(B, H, Hkv, N, d, dv, causal, block, dt, True)
    ws = workspace if workspace is not None else _workspace(need, q.device, stream)
    _check_workspace(ws, need, q.device)
    _raise(la2_backward_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dvv), B,
                            H, Hkv, N, d, dv, int(causal), block, dt, _ptr(ws),
                            ws.numel() if ws is not None else 0, _stream_handle(stream)))
    return dq, dk, dvv


def workspace_bytes_decay(B, H, N, d, dv, block, dtype_code, is_backward) -> int:
    n = la2_workspace_size_decay(B, H, N, d, dv, block, dtype_code, int(is_backward))
    if n == ctypes.c_size_t(-1).value:
        raise La2Error(LA2_ERR_INVALID_ARG)
    return int(n)


def _decay_rates(lam, q, stream):
    """Per-head rates as a float32 CUDA tensor of H values on q's device (a
    copy, when one is needed, is made on the stream the kernels run on)."""
    import torch

    lam = torch.as_tensor(lam, dtype=torch.float32).reshape(-1)
    if lam.numel() != q.shape[1]:
        raise La2Error(LA2_ERR_INVALID_ARG)
    if stream is None:
        return lam.to(q.device).contiguous()
    with torch.cuda.stream(stream):
        return lam.to(q.device).contiguous()


def forward_decay(q, k, v, lam, block: int = 64, out=None, workspace=None, stream=None):
    """Decayed causal form: o_t = sum_{s<=t} lam_h^(t-s) (q_t . k_s) v_s for
    [B,H,N,d] CUDA tensors and H per-head rates ``lam``; returns O."""
    import torch

    _check_inputs(q, k, v)
    if q.dim() != 4:
        raise La2Error(LA2_ERR_INVALID_ARG)
    B, H, N, d = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    _check_like(q, q.shape, q.dtype, k)
    _check_like(q, (B, H, N, dv), q.dtype, v)
    rates = _decay_rates(lam, q, stream)
    if out is None:
        out = torch.empty((B, H, N, dv), dtype=q.dtype, device=q.device)
    _check_inputs(out)
    _check_like(q, (B, H, N, dv), q.dtype, out)
    need = workspace_bytes_decay(B, H, N, d, dv, block, dt, False)
    ws = workspace if workspace is not None else _workspace(need, q.device, stream)
    _check_workspace(ws, need, q.device)
    _raise(la2_forward_decay(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(rates), B, H, N, d, dv,
                             block, dt, _ptr(ws), ws.numel() if ws is not None else 0,
                             _stream_handle(stream)))
    return out


def backward_decay(q, k, v, do, lam, block: int = 64, outs=None, workspace=None, stream=None):
    """Gradients (dQ, dK, dV) of <dO, O> for the decayed causal form."""
    import torch

    _check_inputs(q, k, v, do)
    if q.dim() != 4:
        raise La2Error(LA2_ERR_INVALID_ARG)
    B, H, N, d = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    _check_like(q, q.shape, q.dtype, k)
    _check_like(q, (B, H, N, dv), q.dtype, v, do)
    rates = _decay_rates(lam, q, stream)
    if outs is None:
        outs = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    dq, dk, dvv = outs
    _check_inputs(dq, dk, dvv)
    _check_like(q, q.shape, q.dtype, dq, dk)
    _check_like(q, (B, H, N, dv), q.dtype, dvv)
    need = workspace_bytes_decay(B, H, N, d, dv, block, dt, True)
    ws = workspace if workspace is not None else _workspace(need, q.device, stream)
    _check_workspace(ws, need, q.device)
    _raise(la2_backward_decay(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dvv),
                              _ptr(rates), B, H, N, d, dv, block, dt, _ptr(ws),
                              ws.numel() if ws is not None else 0, _stream_handle(stream)))
    return dq, dk, dvv


def kv_state(k, v, state=None, workspace=None, stream=None):
    """state += sum_t k_t^T v_t per sequence; k [B,H,N,d], v [B,H,N,dv] CUDA
    tensors, state [B,H,d,dv] float32 (zeros if omitted). Returns the state."""
    import torch

    _check_inputs(k, v)
    if k.dim() != 4 or v.dim() != 4:
        raise La2Error(LA2_ERR_INVALID_ARG)
    B, H, N, d = k.shape
    dv = v.shape[-1]
    dt = _dtype_code(k)
    _check_like(k, (B, H, N, dv), k.dtype, v)
    if state is None:
        state = torch.zeros((B, H, d, dv), dtype=torch.float32, device=k.device)
    _check_inputs(state)
    _check_like(k, (B, H, d, dv), torch.float32, state)
    need = la2_kv_state_workspace_size(B, H, N, d, dv, dt)
    if need == ctypes.c_size_t(-1).value:
        raise La2Error(LA2_ERR_INVALID_ARG)
    ws = workspace if workspace is not None else _workspace(need, k.device, stream)
    _check_workspace(ws, need, k.device)
    _raise(la2_kv_state(_ptr(k), _ptr(v), _ptr(state), B, H, N, d, dv, dt, _ptr(ws),
                        ws.numel() if ws is not None else 0, _stream_handle(stream)))
    return state


def decode_step(q, k, v, state, out=None, stream=None):
    """One RNN-mode token per sequence: state += k^T v, o = q state. q, k [B,H,d],
    v [B,H,dv] CUDA tensors, state [B,H,d,dv] float32 (updated in place). Returns o."""
    import torch

    _check_inputs(q, k, v, state)
    if q.dim() != 3 or v.dim() != 3:
        raise La2Error(LA2_ERR_INVALID_ARG)
    B, H, d = q.shape
    dv = v.shape[-1]
    _dtype_code(q)
    _check_like(q, q.shape, q.dtype, k)
    _check_like(q, (B, H, dv), q.dtype, v)
    _check_like(q, (B, H, d, dv), torch.float32, state)
    if out is None:
        out = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    _check_inputs(out)
    _check_like(q, (B, H, dv), q.dtype, out)
    _raise(la2_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(state), B, H, d, dv,
                           _dtype_code(q), _stream_handle(stream)))
    return out


def check(stream=None):
    _raise(la2_check(_stream_handle(stream)))


def _states_arg(states, q):
    """(pointer, count) of a [n,B,H,d,dv] float32 stack of states (None: none)."""
    import torch

    if states is None or states.shape[0] == 0:
        return _vp(0), 0
    B, H, _, d = q.shape
    _check_inputs(states)
    if states.dim() != 5 or tuple(states.shape[1:4]) != (B, H, d) or states.dtype != torch.float32 \
            or states.device != q.device:
        raise La2Error(LA2_ERR_INVALID_ARG)
    return _ptr(states), int(states.shape[0])


def forward_sp(q, k, v, prefix_states=None, block: int = 64, out=None, workspace=None, stream=None):
    """Causal output of one part of longer sequences: ``prefix_states``
    [n,B,H,d,dv] float32 sum to the KV state of everything before the part."""
    import torch

    _check_inputs(q, k, v)
    if q.dim() != 4 or v.dim() != 4:
        raise La2Error(LA2_ERR_INVALID_ARG)
    B, H, N, d = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    _check_like(q, q.shape, q.dtype, k)
    _check_like(q, (B, H, N, dv), q.dtype, v)
    if out is None:
        out = torch.empty((B, H, N, dv), dtype=q.dtype, device=q.device)
    _check_inputs(out)
    _check_like(q, (B, H, N, dv), q.dtype, out)
    pp, npre = _states_arg(prefix_states, q)
    need = la2_workspace_size_sp(B, H, N, d, dv, block, dt, 0)
    if need == ctypes.c_size_t(-1).value:
        raise La2Error(LA2_ERR_INVALID_ARG)
    ws = workspace if workspace is not None else _workspace(need, q.device, stream)
    _check_workspace(ws, need, q.device)
    _raise(la2_forward_sp(_ptr(q), _ptr(k), _ptr(v), _ptr(out), pp, npre, B, H, N, d, dv, block, dt,
                          _ptr(ws), ws.numel() if ws is not None else 0, _stream_handle(stream)))
    return out


def backward_sp(q, k, v, do, prefix_states=None, suffix_states=None, block: int = 64, outs=None,
                workspace=None, stream=None):
    """Gradients of one part of longer sequences: ``prefix_states`` sum to the
    KV state before the part, ``suffix_states`` to sum q^T dO after it."""
    import torch

    _check_inputs(q, k, v, do)
    if q.dim() != 4 or v.dim() != 4:
        raise La2Error(LA2_ERR_INVALID_ARG)
    B, H, N, d = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    _check_like(q, q.shape, q.dtype, k)
    _check_like(q, (B, H, N, dv), q.dtype, v, do)
    if outs is None:
        outs = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    dq, dk, dvv = outs
    _check_inputs(dq, dk, dvv)
    _check_like(q, q.shape, q.dtype, dq, dk)
    _check_like(q, (B, H, N, dv), q.dtype, dvv)
    pp, npre = _states_arg(prefix_states, q)
    sp, nsuf = _states_arg(suffix_states, q)
    need = la2_workspace_size_sp(B, H, N, d, dv, block, dt, 1)
    if need == ctypes.c_size_t(-1).value:
        raise La2Error(LA2_ERR_INVALID_ARG)
    ws = workspace if workspace is not None else _workspace(need, q.device, stream)
    _check_workspace(ws, need, q.device)
    _raise(la2_backward_sp(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dvv), pp,
                           npre, sp, nsuf, B, H, N, d, dv, block, dt, _ptr(ws),
                           ws.numel() if ws is not None else 0, _stream_handle(stream)))
    return dq, dk, dvv
