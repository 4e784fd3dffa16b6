"""The C-ABI library loads, exports every symbol include/ttt.h declares, and
rejects bad arguments on the host with the documented status codes.

Every call here carries at least one argument error, so validation returns
before anything is launched; the pointer values are never dereferenced.
No GPU is needed.
"""
from __future__ import annotations

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ttt.h")

b = pytest.importorskip("test_sequence_layers_ttt_b200._binding")

OK, NULL, SHAPE, DTYPE, ALIGN, ALIAS, UNSUP = 0, 1, 2, 3, 4, 5, 6


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:ttt_status|ttt_impl|const char\*|int|size_t)\s+(ttt_\w+)\s*\(",
                                 text, re.M)))


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("ttt_linear_forward", "ttt_mlp_forward", "ttt_status_string",
              "ttt_linear_forward_impl", "ttt_abi_version", "ttt_linear_pick_impl"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(b.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/ttt.h but not exported"


def test_status_strings():
    for code, name in enumerate(b.STATUS):
        assert b.status_string(code).startswith(name)
    assert b.status_string(99) == "TTT_ERR_UNKNOWN"
    assert b.lib.ttt_abi_version() == 103


# Fake, 16-byte aligned, non-overlapping device addresses.  Never dereferenced:
# every case below fails validation first.
BASE = 1 << 40
STRIDE = 1 << 34


def fake(i):
    return BASE + i * STRIDE


def linear_call(B=1, H=2, T=64, d=64, mb=16, dtype=0, mode=0, eps=1e-6, ptrs=None, impl=0):
    p = [fake(i) for i in range(11)] if ptrs is None else ptrs
    return b.lib.ttt_linear_forward_impl(B, H, T, d, mb, dtype, mode, eps, *p, impl, None)


def mlp_call(B=1, H=2, T=64, d=64, hid=256, mb=16, dtype=0, eps=1e-6, ptrs=None):
    p = [fake(i) for i in range(15)] if ptrs is None else ptrs
    return b.lib.ttt_mlp_forward(B, H, T, d, hid, mb, dtype, eps, *p, None)


def with_ptr(i, value, n=11):
    p = [fake(k) for k in range(n)]
    p[i] = value
    return p


# argument order: Q K V eta W0 b0 gamma beta Z W_T b_T
@pytest.mark.parametrize("idx", [0, 1, 2, 3, 4, 8, 9])
def test_linear_null_required_pointer(idx):
    assert linear_call(ptrs=with_ptr(idx, None)) == NULL


@pytest.mark.parametrize("idx", [5, 6, 7, 10])
def test_linear_ln_mode_needs_bias_and_ln_params(idx):
    assert linear_call(ptrs=with_ptr(idx, None)) == NULL


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), SHAPE), (dict(H=0), SHAPE), (dict(T=-1), SHAPE), (dict(mb=0), SHAPE),
    (dict(mb=12), SHAPE), (dict(mb=24), SHAPE), (dict(mb=3), SHAPE),
    (dict(eps=0.0), SHAPE), (dict(eps=-1.0), SHAPE),
    (dict(dtype=7), DTYPE), (dict(d=48), UNSUP), (dict(d=128), UNSUP), (dict(mode=5), UNSUP),
    (dict(B=1 << 16, H=1 << 16), SHAPE),
])
def test_linear_bad_shapes(kw, code):
    assert linear_call(**kw) == code


@pytest.mark.parametrize("idx", range(11))
def test_linear_misaligned_pointer(idx):
    assert linear_call(ptrs=with_ptr(idx, fake(idx) + 8)) == ALIGN


def test_linear_z_overlapping_q_is_alias():
    p = [fake(k) for k in range(11)]
    p[8] = p[0] + 256  # Z inside Q
    assert linear_call(ptrs=p) == ALIAS


def test_linear_partial_state_overlap_is_alias():
    p = [fake(k) for k in range(11)]
    p[9] = p[4] + 16  # W_T overlaps W0 but is not the same pointer
    assert linear_call(ptrs=p) == ALIAS


def test_linear_outputs_overlapping_each_other_is_alias():
    p = [fake(k) for k in range(11)]
    p[10] = p[8] + 64  # b_T inside Z
    assert linear_call(ptrs=p) == ALIAS


# MLP: Q K V eta W1 b1 W2 b2 gamma beta Z W1_T b1_T W2_T b2_T
@pytest.mark.parametrize("idx", range(15))
def test_mlp_null_pointer(idx):
    assert mlp_call(ptrs=with_ptr(idx, None, 15)) == NULL


@pytest.mark.parametrize("kw,code", [
    (dict(d=32), UNSUP), (dict(hid=128), UNSUP), (dict(mb=10), SHAPE), (dict(B=0), SHAPE),
    (dict(dtype=3), DTYPE), (dict(eps=0.0), SHAPE)])
def test_mlp_bad_shapes(kw, code):
    assert mlp_call(**kw) == code


def test_mlp_alias_and_align():
    p = [fake(k) for k in range(15)]
    p[10] = p[2] + 1024  # Z inside V
    assert mlp_call(ptrs=p) == ALIAS
    assert mlp_call(ptrs=with_ptr(13, fake(13) + 4, 15)) == ALIGN


# decode: Q K V eta W b W_mb b_mb gamma beta Z
def decode_call(B=1, H=2, T=64, d=64, mb=16, pos0=0, dtype=0, mode=0, eps=1e-6, ptrs=None):
    p = [fake(i) for i in range(11)] if ptrs is None else ptrs
    return b.lib.ttt_linear_decode(B, H, T, d, mb, pos0, dtype, mode, eps, *p, None)


@pytest.mark.parametrize("pos0", [-1, 16, 100])
def test_decode_position_outside_the_mini_batch(pos0):
    assert decode_call(pos0=pos0) == SHAPE


def test_decode_bad_mini_batch():
    assert decode_call(mb=12) == SHAPE


@pytest.mark.parametrize("idx", [4, 6, 7, 8, 9])
def test_decode_null_state_or_ln_params(idx):
    assert decode_call(ptrs=with_ptr(idx, None)) == NULL


@pytest.mark.parametrize("idx", [4, 5, 6, 7, 10])
def test_decode_misaligned_state_or_output(idx):
    assert decode_call(ptrs=with_ptr(idx, fake(idx) + 4)) == ALIGN


@pytest.mark.parametrize("dst,src,off", [(6, 4, 64), (6, 10, 0), (7, 0, 128), (4, 6, 16), (10, 5, 0)])
def test_decode_overlapping_buffers(dst, src, off):
    p = [fake(k) for k in range(11)]
    p[dst] = p[src] + off
    assert decode_call(ptrs=p) == ALIAS


# MLP decode: Q K V eta W1 b1 W2 b2 W1_mb b1_mb W2_mb b2_mb gamma beta Z
def mlp_decode_call(B=1, H=2, T=64, mb=16, pos0=0, ptrs=None):
    p = [fake(i) for i in range(15)] if ptrs is None else ptrs
    return b.lib.ttt_mlp_decode(B, H, T, 64, 256, mb, pos0, 0, 1e-6, *p, None)


@pytest.mark.parametrize("pos0", [-1, 16])
def test_mlp_decode_position_outside_the_mini_batch(pos0):
    assert mlp_decode_call(pos0=pos0) == SHAPE


@pytest.mark.parametrize("idx", [4, 8, 9, 10, 11])
def test_mlp_decode_null_state(idx):
    assert mlp_decode_call(ptrs=with_ptr(idx, None, 15)) == NULL


@pytest.mark.parametrize("idx", [8, 9, 10, 11])
def test_mlp_decode_misaligned_start_state(idx):
    assert mlp_decode_call(ptrs=with_ptr(idx, fake(idx) + 4, 15)) == ALIGN


@pytest.mark.parametrize("dst,src,off", [(8, 4, 256), (11, 14, 0), (10, 0, 64), (9, 5, 0)])
def test_mlp_decode_overlapping_buffers(dst, src, off):
    p = [fake(k) for k in range(15)]
    p[dst] = p[src] + off
    assert mlp_decode_call(ptrs=p) == ALIAS


@pytest.mark.parametrize("impl", [2, 3, 9])
def test_mlp_decode_families(impl):
    # decode has the decode kernel (auto) and the generic scan; other families are
    # refused after validation, before any launch
    p = [fake(i) for i in range(15)]
    assert b.lib.ttt_mlp_decode_impl(1, 2, 64, 64, 256, 16, 0, 0, 1e-6, *p, impl, None) == UNSUP


def test_linear_has_no_split_family():
    # the split family is TTT-MLP only; unknown families are refused before any launch
    assert linear_call(impl=3) == UNSUP
    assert linear_call(impl=9) == UNSUP


def test_pick_impl_is_a_host_query():
    f = b.lib.ttt_linear_pick_impl
    assert f(1, 2, 64, 16, 16, 1, 0) == 1        # fp32 d=16: generic
    assert f(1, 2, 64, 48, 16, 0, 0) == 0        # d=48: nothing
    assert f(2, 32, 32768, 64, 16, 0, 0) in (1, 2)


@pytest.mark.parametrize("B,H,n", [(1, 3, 8), (2, 32, 8), (4, 12, 8), (2, 5, 8), (1, 1, 8), (3, 7, 4)])
def test_host_pipeline_groups_cover_every_scan_once(B, H, n):
    from test_sequence_layers_ttt_b200 import _binding as ttt
    groups = ttt._head_groups(B, H, n)
    seen = [(b, h) for b, h0, h1 in groups for h in range(h0, h1)]
    assert sorted(seen) == [(b, h) for b in range(B) for h in range(H)]
    assert all(h1 > h0 for _, h0, h1 in groups)


def test_mlp_pick_impl_is_a_host_query():
    from test_sequence_layers_ttt_b200 import _binding as ttt
    # two SMs per scan while 2 B H CTAs fit in one wave, one SM per scan beyond
    assert ttt.mlp_pick_impl(4, 12, 8192, 64, 256, 16, "bf16") == "tensorcore_split"
    assert ttt.mlp_pick_impl(4, 16, 8192, 64, 256, 16, "bf16") == "tensorcore_split"
    assert ttt.mlp_pick_impl(2, 37, 8192, 64, 256, 16, "bf16") == "tensorcore_split"
    assert ttt.mlp_pick_impl(5, 15, 8192, 64, 256, 16, "bf16") == "tensorcore"
    assert ttt.mlp_pick_impl(8, 32, 2048, 64, 256, 16, "bf16") == "tensorcore"
    assert ttt.mlp_pick_impl(4, 12, 8192, 64, 256, 16, "f32") == "generic"
    assert ttt.mlp_pick_impl(4, 12, 8192, 64, 256, 32, "bf16") == "generic"
    assert ttt.mlp_pick_impl(4, 12, 8200, 64, 256, 16, "bf16") == "generic"
    assert ttt.mlp_pick_impl(4, 12, 8192, 64, 128, 16, "bf16") == "none"


def test_empty_sequence_allows_null_token_buffers_but_not_state():
    p = [fake(k) for k in range(11)]
    for i in (0, 1, 2, 3, 8):
        p[i] = None
    p[4] = None  # W0 is still required
    assert linear_call(T=0, ptrs=p) == NULL


# ---------------------------------------------------------------- layer backward (host validation only)
# argument order: Q K V eta W0 b0 gamma beta dZ dW_T db_T dQ dK dV deta dW0 db0 dgamma dbeta workspace
def backward_call(B=1, H=2, T=64, d=64, mb=16, dtype=0, mode=0, eps=1e-6, ptrs=None, ws_bytes=None):
    p = [fake(i) for i in range(20)] if ptrs is None else ptrs
    need = b.lib.ttt_linear_backward_workspace_size(B, H, T, d, mb)
    ws = need if ws_bytes is None else ws_bytes
    return b.lib.ttt_linear_backward(B, H, T, d, mb, dtype, mode, eps, *p, ctypes.c_size_t(ws), None)


def test_backward_workspace_size_formula():
    B, H, T, d, mb = 2, 3, 40, 64, 16
    nmb = -(-T // mb)
    assert b.linear_backward_workspace_size(B, H, T, d, mb) == 4 * (B * H * nmb * (d * d + d) + B * H * 2 * d)
    assert b.linear_backward_workspace_size(0, 1, 1, 64, 16) == 0


@pytest.mark.parametrize("idx", [0, 1, 2, 3, 4, 5, 6, 7, 8, 11, 12, 13, 14, 15, 16, 17, 18, 19])
def test_backward_null_required_pointer(idx):
    p = [fake(k) for k in range(20)]
    p[idx] = None
    expected = b.STATUS.index("TTT_ERR_WORKSPACE") if idx == 19 else NULL
    assert backward_call(ptrs=p) == expected


def test_backward_state_gradients_may_be_null_and_workspace_is_checked():
    p = [fake(k) for k in range(20)]
    p[9] = p[10] = None
    assert backward_call(ptrs=p, ws_bytes=16) == b.STATUS.index("TTT_ERR_WORKSPACE")


@pytest.mark.parametrize("kw,code", [
    (dict(mode=1), UNSUP), (dict(mb=32), UNSUP), (dict(d=48), UNSUP), (dict(mb=0), SHAPE), (dict(B=0), SHAPE),
    (dict(dtype=4), DTYPE), (dict(eps=0.0), SHAPE)])
def test_backward_bad_shapes(kw, code):
    assert backward_call(**kw) == code


def test_backward_alias_and_align():
    p = [fake(k) for k in range(20)]
    p[11] = p[8] + 256  # dQ inside dZ
    assert backward_call(ptrs=p) == ALIAS
    p = [fake(k) for k in range(20)]
    p[15] = p[19] + 64  # dW0 inside the workspace
    assert backward_call(ptrs=p) == ALIAS
    p = [fake(k) for k in range(20)]
    p[14] = fake(14) + 4
    assert backward_call(ptrs=p) == ALIGN
