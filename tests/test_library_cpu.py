"""Host-only checks of libla2.so: it loads, exports what include/la2.h declares,
and rejects bad arguments before touching the device (no GPU needed)."""

import ctypes
import os
import re

import pytest

from linear_attention_la2_b200 import build as la2_build

la2_build.build()
from linear_attention_la2_b200 import la2  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NULL = ctypes.c_void_p(0)


def declared_symbols():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            text = open(os.path.join(inc, f)).read()
            names.update(re.findall(r"LA2_API[^;(]*?\b(la2_\w+)\s*\(", text))
    return sorted(names)


def test_header_declares_entry_points():
    names = declared_symbols()
    for required in ("la2_forward", "la2_backward", "la2_workspace_size", "la2_check",
                     "la2_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(la2.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert name in la2.EXPORTED, name


def test_status_strings():
    for code in range(6):
        s = la2.la2_status_string(code)
        assert s.startswith("LA2_")
    assert "unknown" in la2.la2_status_string(99)


def _fwd(**kw):
    args = dict(q=NULL, k=NULL, v=NULL, o=NULL, B=1, H=1, N=16, d=64, dv=64, causal=1, block=64,
                dt=la2.LA2_F32, ws=NULL, wsb=0, stream=NULL)
    args.update(kw)
    return la2.la2_forward(args["q"], args["k"], args["v"], args["o"], args["B"], args["H"],
                           args["N"], args["d"], args["dv"], args["causal"], args["block"],
                           args["dt"], args["ws"], args["wsb"], args["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(B=-1), la2.LA2_ERR_INVALID_ARG),
    (dict(N=-5), la2.LA2_ERR_INVALID_ARG),
    (dict(d=0), la2.LA2_ERR_INVALID_ARG),
    (dict(dv=0), la2.LA2_ERR_INVALID_ARG),
    (dict(causal=2), la2.LA2_ERR_INVALID_ARG),
    (dict(dt=7), la2.LA2_ERR_INVALID_ARG),
    (dict(block=0), la2.LA2_ERR_INVALID_ARG),
    (dict(block=48), la2.LA2_ERR_UNSUPPORTED),
    (dict(d=129), la2.LA2_ERR_UNSUPPORTED),
    (dict(dt=la2.LA2_BF16, d=96), la2.LA2_ERR_UNSUPPORTED),
    (dict(dt=la2.LA2_BF16, block=32), la2.LA2_ERR_UNSUPPORTED),
    (dict(d=128, dv=128, block=128), la2.LA2_ERR_UNSUPPORTED),  # fp32 tiles exceed smem
    (dict(), la2.LA2_ERR_INVALID_ARG),  # NULL pointers
    (dict(q=ctypes.c_void_p(0x1008), k=ctypes.c_void_p(0x2000), v=ctypes.c_void_p(0x3000),
          o=ctypes.c_void_p(0x4000)), la2.LA2_ERR_INVALID_ARG),  # q not 16-byte aligned
    (dict(q=ctypes.c_void_p(0x10000), k=ctypes.c_void_p(0x20000), v=ctypes.c_void_p(0x30000),
          o=ctypes.c_void_p(0x10100)), la2.LA2_ERR_INVALID_ARG),  # o overlaps q
])
def test_forward_rejects_bad_arguments(kw, code):
    assert _fwd(**kw) == code


def test_empty_problem_is_a_noop():
    for kw in (dict(B=0), dict(H=0), dict(N=0)):
        assert _fwd(**kw) == la2.LA2_OK
        assert la2.la2_workspace_size(kw.get("B", 1), kw.get("H", 1), kw.get("N", 16), 64, 64, 1,
                                      64, la2.LA2_F32, 0) == 0


def test_backward_rejects_bad_arguments():
    b = la2.la2_backward
    assert b(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, 1, 16, 64, 64, 1, 64, la2.LA2_F32, NULL, 0,
             NULL) == la2.LA2_ERR_INVALID_ARG
    assert b(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, 1, 16, 64, 64, 3, 64, la2.LA2_F32, NULL, 0,
             NULL) == la2.LA2_ERR_INVALID_ARG
    assert b(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, 1, 16, 64, 64, 1, 64, la2.LA2_F32, NULL, 0,
             NULL) == la2.LA2_OK
    p = [ctypes.c_void_p(0x100000 * (i + 1)) for i in range(7)]
    p[4] = ctypes.c_void_p(0x100000 + 64)  # dq overlaps q
    assert b(*p, 1, 1, 16, 64, 64, 1, 64, la2.LA2_F32, NULL, 0, NULL) == la2.LA2_ERR_INVALID_ARG


def test_workspace_size_rejects_bad_arguments():
    bad = ctypes.c_size_t(-1).value
    assert la2.la2_workspace_size(1, 1, 16, 64, 64, 5, 64, la2.LA2_F32, 0) == bad
    assert la2.la2_plan_ranges(1, 1, 16, 128, 128, 1, 48, la2.LA2_BF16, 0, None, 0) == -1


def test_settings_validation():
    assert la2.la2_set_chunk_len(-1) == la2.LA2_ERR_INVALID_ARG
    assert la2.la2_set_chunk_len(0) == la2.LA2_OK
    assert la2.la2_set_spin_limit(-3) == la2.LA2_ERR_INVALID_ARG
    assert la2.la2_set_spin_limit(0) == la2.LA2_OK


def test_profiler_names():
    n = la2.la2_profile_num_kernels()
    assert n >= 5
    names = [la2.la2_profile_kernel_name(i) for i in range(n)]
    assert all(names) and len(set(names)) == n
    assert la2.la2_profile_kernel_name(n) == ""
    assert la2.la2_version() > 0
    assert la2.la2_profile_enable(3) == la2.LA2_ERR_INVALID_ARG
    for on in (1, 0, 2, 0):
        assert la2.la2_profile_enable(on) == la2.LA2_OK


def _dec(**kw):
    a = dict(q=NULL, k=NULL, v=NULL, o=NULL, s=NULL, B=1, H=2, d=64, dv=32, dt=la2.LA2_BF16)
    a.update(kw)
    return la2.la2_decode_step(a["q"], a["k"], a["v"], a["o"], a["s"], a["B"], a["H"], a["d"],
                               a["dv"], a["dt"], NULL)


def test_decode_step_rejects_bad_arguments():
    P = [ctypes.c_void_p(0x100000 * (i + 1)) for i in range(5)]
    ok = dict(q=P[0], k=P[1], v=P[2], o=P[3], s=P[4])
    assert _dec() == la2.LA2_ERR_INVALID_ARG                     # NULL pointers
    assert _dec(B=0) == la2.LA2_OK                               # empty problem
    assert _dec(d=0, **ok) == la2.LA2_ERR_INVALID_ARG
    assert _dec(dv=-1, **ok) == la2.LA2_ERR_INVALID_ARG
    assert _dec(dt=9, **ok) == la2.LA2_ERR_INVALID_ARG
    assert _dec(**dict(ok, q=ctypes.c_void_p(0x100001))) == la2.LA2_ERR_INVALID_ARG  # misaligned
    assert _dec(**dict(ok, s=ctypes.c_void_p(0x100002))) == la2.LA2_ERR_INVALID_ARG  # state misaligned
    assert _dec(**dict(ok, o=ctypes.c_void_p(0x100000 + 64))) == la2.LA2_ERR_INVALID_ARG  # o overlaps q
    # the state (2*64*32*4 = 16 KiB) overlaps v when placed just before it
    assert _dec(**dict(ok, s=ctypes.c_void_p(0x300000 - 4096))) == la2.LA2_ERR_INVALID_ARG


def test_kv_state_rejects_bad_arguments():
    ks = la2.la2_kv_state
    bad = ctypes.c_size_t(-1).value
    assert la2.la2_kv_state_workspace_size(1, 1, 16, 64, 64, 7) == bad
    assert la2.la2_kv_state_workspace_size(1, 1, 16, 96, 64, la2.LA2_BF16) == bad
    assert la2.la2_kv_state_workspace_size(0, 1, 16, 64, 64, la2.LA2_F32) == 0
    assert ks(NULL, NULL, NULL, 1, 1, 16, 64, 64, la2.LA2_F32, NULL, 0, NULL) == la2.LA2_ERR_INVALID_ARG
    assert ks(NULL, NULL, NULL, 1, 0, 16, 64, 64, la2.LA2_F32, NULL, 0, NULL) == la2.LA2_OK
    assert ks(NULL, NULL, NULL, 1, 1, -2, 64, 64, la2.LA2_F32, NULL, 0, NULL) == la2.LA2_ERR_INVALID_ARG
    P = [ctypes.c_void_p(0x1000000 * (i + 1)) for i in range(3)]
    # state overlapping k
    assert ks(P[0], P[1], ctypes.c_void_p(0x1000000 + 256), 1, 1, 16, 64, 64, la2.LA2_F32, NULL, 0,
              NULL) == la2.LA2_ERR_INVALID_ARG


def test_binding_rejects_mismatched_tensors():
    """The binding checks every tensor against q before the library sizes its
    tensor maps from q's shape (a shorter k, v or output would be read or
    written past its end)."""
    import torch

    q = torch.zeros(1, 2, 16, 64)
    la2._check_like(q, q.shape, q.dtype, torch.zeros(1, 2, 16, 64))
    for bad in (torch.zeros(1, 2, 15, 64), torch.zeros(2, 2, 16, 64), torch.zeros(1, 2, 16, 32),
                torch.zeros(1, 2, 16, 64, dtype=torch.bfloat16)):
        with pytest.raises(la2.La2Error) as e:
            la2._check_like(q, q.shape, q.dtype, bad)
        assert e.value.code == la2.LA2_ERR_INVALID_ARG
    # host tensors are rejected before anything reaches the library
    for fn, args in ((la2.forward, (q, q, q)), (la2.backward, (q, q, q, q)),
                     (la2.kv_state, (q, q)), (la2.decode_step, (q[0], q[0], q[0], q))):
        with pytest.raises(la2.La2Error):
            fn(*args)
    with pytest.raises(la2.La2Error) as e:
        la2._check_workspace(None, 256, None)
    assert e.value.code == la2.LA2_ERR_WORKSPACE


def test_header_states_the_tensor_core_shapes():
    """The header's supported-shape text matches the dispatch: bf16 runs on the
    tensor cores only at d = dv = 128."""
    text = open(os.path.join(ROOT, "include", "la2.h")).read()
    assert "d = dv = 128 runs on the tensor cores" in text
    src = open(os.path.join(ROOT, "linear_attention_la2_b200", "csrc", "la2_sm100.cuh")).read()
    assert "return d == 128 && dv == 128 && (block == 64 || block == 128);" in src
    # bf16 shapes off the tensor-core path are accepted (pointer check fails first)
    assert _fwd(dt=la2.LA2_BF16, d=64, dv=128) == la2.LA2_ERR_INVALID_ARG
    assert _fwd(dt=la2.LA2_BF16, d=128, dv=64, block=128) == la2.LA2_ERR_INVALID_ARG


def test_gqa_rejects_bad_head_counts():
    """H must be a multiple of the K/V head count Hkv >= 1."""
    bad = ctypes.c_size_t(-1).value
    ws = la2.la2_workspace_size_gqa
    for H, Hkv in ((8, 3), (8, 0), (8, -1), (4, 8)):
        assert ws(1, H, Hkv, 16, 64, 64, 1, 64, la2.LA2_F32, 0) == bad
        assert la2.la2_forward_gqa(NULL, NULL, NULL, NULL, 1, H, Hkv, 16, 64, 64, 1, 64, la2.LA2_F32,
                                   NULL, 0, NULL) == la2.LA2_ERR_INVALID_ARG
        assert la2.la2_backward_gqa(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, H, Hkv, 16, 64, 64,
                                    1, 64, la2.LA2_F32, NULL, 0, NULL) == la2.LA2_ERR_INVALID_ARG
    # empty problems are still no-ops
    assert la2.la2_forward_gqa(NULL, NULL, NULL, NULL, 0, 8, 2, 16, 64, 64, 1, 64, la2.LA2_F32, NULL,
                               0, NULL) == la2.LA2_OK
    assert ws(1, 0, 0, 16, 64, 64, 1, 64, la2.LA2_F32, 0) == 0
    # a valid grouping with NULL pointers fails only on the pointers
    assert la2.la2_forward_gqa(NULL, NULL, NULL, NULL, 1, 8, 2, 16, 64, 64, 1, 64, la2.LA2_F32, NULL,
                               0, NULL) == la2.LA2_ERR_INVALID_ARG


def test_binding_checks_grouped_shapes():
    import torch

    q = torch.zeros(1, 8, 16, 64)
    assert la2._kv_heads(q, torch.zeros(1, 2, 16, 64), torch.zeros(1, 2, 16, 64)) == 2
    for kv in (torch.zeros(1, 3, 16, 64), torch.zeros(1, 0, 16, 64)):
        with pytest.raises(la2.La2Error):
            la2._kv_heads(q, kv, kv)


def _fwd_decay(**kw):
    args = dict(q=NULL, k=NULL, v=NULL, o=NULL, lam=NULL, B=1, H=1, N=16, d=64, dv=64, block=64,
                dt=la2.LA2_F32, ws=NULL, wsb=0, stream=NULL)
    args.update(kw)
    return la2.la2_forward_decay(args["q"], args["k"], args["v"], args["o"], args["lam"], args["B"],
                                 args["H"], args["N"], args["d"], args["dv"], args["block"],
                                 args["dt"], args["ws"], args["wsb"], args["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(B=-1), la2.LA2_ERR_INVALID_ARG),
    (dict(d=0), la2.LA2_ERR_INVALID_ARG),
    (dict(dt=7), la2.LA2_ERR_INVALID_ARG),
    (dict(d=200), la2.LA2_ERR_UNSUPPORTED),
    (dict(block=48), la2.LA2_ERR_UNSUPPORTED),
    (dict(B=0), la2.LA2_OK),
    # valid shape, missing tensors or rates
    (dict(), la2.LA2_ERR_INVALID_ARG),
    (dict(q=4096, k=8192, v=12288, o=16384), la2.LA2_ERR_INVALID_ARG),  # no rates
    (dict(q=4096, k=8192, v=12288, o=16384, lam=16386), la2.LA2_ERR_INVALID_ARG),  # misaligned rates
    (dict(q=4096, k=8192, v=12288, o=16384, lam=16384), la2.LA2_ERR_INVALID_ARG),  # rates inside o
])
def test_forward_decay_rejects_bad_arguments(kw, code):
    assert _fwd_decay(**kw) == code


def test_backward_decay_limits():
    """bf16 d = dv = 128 runs both ways on tensor cores, at block 64 and 128 (the
    shape passes; here only the missing tensors are refused). Off those shapes
    the backward runs on CUDA cores with their shared-memory limits: f32 d = dv =
    128 at block 128 does not fit the dK/dV tiles (documented in la2.h)."""
    bf, f32 = la2.LA2_BF16, la2.LA2_F32
    for block in (64, 128):
        assert la2.la2_backward_decay(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, 1, 16, 128,
                                      128, block, bf, NULL, 0, NULL) == la2.LA2_ERR_INVALID_ARG
    assert la2.la2_backward_decay(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, 1, 16, 128, 128,
                                  128, f32, NULL, 0, NULL) == la2.LA2_ERR_UNSUPPORTED
    assert la2.la2_workspace_size_decay(1, 1, 16, 128, 128, 128, f32, 1) == ctypes.c_size_t(-1).value
    assert la2.la2_backward_decay(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, 1, 16, 128, 128,
                                  64, bf, NULL, 0, NULL) == la2.LA2_OK
    # the tensor-core backward's row reversal indexes B*H*N rows in 32 bits; the
    # forward has no such limit (there only the missing tensors are refused)
    big = 2 ** 31
    assert la2.la2_backward_decay(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, 1, big, 128, 128,
                                  64, bf, NULL, 0, NULL) == la2.LA2_ERR_UNSUPPORTED
    assert la2.la2_backward_decay(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, 1, big - 1, 128,
                                  128, 64, bf, NULL, 0, NULL) == la2.LA2_ERR_INVALID_ARG
    assert _fwd_decay(N=big, d=128, dv=128, dt=bf) == la2.LA2_ERR_INVALID_ARG
    assert "la2_forward_decay" in la2.EXPORTED and "la2_backward_decay" in la2.EXPORTED
