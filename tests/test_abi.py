"""The C ABI without a GPU: libvi.so loads, exports every function include/vi.h
declares, and rejects bad arguments on the host before anything is launched.

Only invalid calls are made here; each one must return its error code from
the host-side checks, so no CUDA work is enqueued (there is no device)."""
import ctypes
import os
import re

import pytest

import clip_temporal_modules_b200 as vi
from clip_temporal_modules_b200 import _binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vi.h")

OK, INVALID, ALIGN, UNSUP = 0, -1, -2, -3


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vi_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    from clip_temporal_modules_b200 import build
    build.build()
    return vi.lib()


def test_every_declared_function_is_exported(L):
    names = declared_functions()
    assert {"vi_dual_attn", "vi_temporal_conv", "vi_groupnorm_global"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings_and_version(L):
    assert L.vi_status_string(0) == b"VI_OK"
    assert L.vi_status_string(-2) == b"VI_ERR_ALIGNMENT"
    assert L.vi_status_string(-5) == b"VI_ERR_DEVICE_TIMEOUT"
    assert L.vi_status_string(7) == b"VI_ERR_UNKNOWN"
    assert L.vi_version() >= 100
    assert vi.launch_count() == 0         # nothing launched without a device


A = 1 << 20          # fake 16-byte-aligned "device" addresses, never dereferenced
B = 1 << 30
Cp = 1 << 31
D = 1 << 32


def attn(L, q=A, k=B, v=Cp, o=D, F=64, N=4, P=2, heads=2, d=64, pre=8, post=8, glob=16,
         f32=False):
    fn = L.vi_dual_attn_f32 if f32 else L.vi_dual_attn
    return fn(q, k, v, o, F, N, P, heads, d, pre, post, glob, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=0), INVALID), (dict(o=0), INVALID),
    (dict(F=0), INVALID), (dict(N=0), INVALID), (dict(P=-1), INVALID), (dict(heads=0), INVALID),
    (dict(F=63), INVALID),                      # F % N != 0
    (dict(pre=17), INVALID),                    # C_pre longer than a clip (L = 16)
    (dict(post=-1), INVALID), (dict(glob=65), INVALID),
    (dict(d=32), UNSUP),
    (dict(q=A + 8), ALIGN), (dict(o=D + 2), ALIGN),
    (dict(o=A + 64), INVALID),                  # out overlaps q
])
def test_attention_rejects(L, kw, expect):
    assert attn(L, **kw) == expect


def test_attention_rejects_f32_too(L):
    assert attn(L, F=10, N=4, f32=True) == INVALID
    assert attn(L, v=Cp + 4, f32=True) == ALIGN


def conv(L, x=A, w=B, b=Cp, y=D, F=64, N=4, P=2, C=64, k=3, f32=False):
    fn = L.vi_temporal_conv_f32 if f32 else L.vi_temporal_conv
    return fn(x, w, b, y, F, N, P, C, k, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(x=0), INVALID), (dict(b=0), INVALID), (dict(F=62), INVALID), (dict(k=2), INVALID),
    (dict(k=0), INVALID), (dict(k=35, F=64, N=4), INVALID),   # halo wider than a clip
    (dict(C=0), INVALID), (dict(C=12), ALIGN),                # 12 bf16 = 24 bytes per row
    (dict(w=B + 4), ALIGN), (dict(y=A), INVALID),             # y aliases x
    (dict(y=B - 64), INVALID),                                # y runs into w
])
def test_conv_rejects(L, kw, expect):
    assert conv(L, **kw) == expect


def test_conv_f32_row_alignment(L):
    assert conv(L, C=6, f32=True) == ALIGN      # 24 bytes per row
    assert conv(L, F=7, N=7, k=3, C=8, f32=True, x=0) == INVALID


def gn(L, x=A, g=B, bt=Cp, y=D, F=64, N=4, P=2, C=64, groups=8, eps=1e-5, f32=False):
    fn = L.vi_groupnorm_global_f32 if f32 else L.vi_groupnorm_global
    return fn(x, g, bt, y, F, N, P, C, groups, eps, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(x=0), INVALID), (dict(groups=0), INVALID), (dict(groups=7), INVALID),
    (dict(eps=-1.0), INVALID), (dict(eps=float("nan")), INVALID), (dict(eps=float("inf")), INVALID),
    (dict(F=65), INVALID), (dict(groups=2048, C=4096), UNSUP),
    (dict(g=B + 8), ALIGN), (dict(C=4, groups=4), ALIGN),
    (dict(y=A + 16), INVALID),                  # partial overlap with x
])
def test_groupnorm_rejects(L, kw, expect):
    assert gn(L, **kw) == expect


def test_binding_signatures_cover_header():
    for n in declared_functions():
        if n not in ("vi_status_string", "vi_launch_count",
                     "vi_temporal_attention_workspace_bytes"):
            assert n in _binding.SIGNATURES, n


E = 1 << 33
G = 1 << 34


def gnconv(L, x=A, g=B, bt=Cp, w=D, b=E, y=G, F=64, N=4, P=2, C=64, groups=8, eps=1e-5, k=3):
    return L.vi_groupnorm_conv(x, g, bt, w, b, y, F, N, P, C, groups, eps, k, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(w=0), INVALID), (dict(groups=7), INVALID), (dict(k=4), INVALID), (dict(F=66), INVALID),
    (dict(eps=-1.0), INVALID), (dict(b=E + 8), ALIGN), (dict(y=A + 32), INVALID),
    (dict(C=40, groups=8), UNSUP),            # no fused kernel for C % 64 != 0
])
def test_groupnorm_conv_rejects(L, kw, expect):
    assert gnconv(L, **kw) == expect


H_ = 1 << 35
I_ = 1 << 36


def tattn(L, x=A, wqkv=B, bqkv=Cp, wo=D, bo=E, out=G, ws=H_, F=64, N=4, P=2, heads=2, d=64,
          pre=8, post=8, glob=16):
    return L.vi_temporal_attention(x, wqkv, bqkv, wo, bo, out, ws, F, N, P, heads, d, pre, post,
                                   glob, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(ws=0), INVALID), (dict(x=0), INVALID), (dict(F=63), INVALID), (dict(pre=17), INVALID),
    (dict(d=32), UNSUP), (dict(ws=H_ + 8), ALIGN),
    (dict(ws=A + 4096), INVALID),             # workspace overlaps x
    (dict(out=H_ + 64), INVALID),             # out inside the workspace
])
def test_temporal_attention_rejects(L, kw, expect):
    assert tattn(L, **kw) == expect


def test_temporal_attention_workspace_bytes(L):
    assert L.vi_temporal_attention_workspace_bytes(1024, 2560, 320) == 4 * 1024 * 2560 * 320 * 2
    assert L.vi_temporal_attention_workspace_bytes(0, 1, 1) == 0


def test_no_global_tuning_state_in_the_abi(L):
    """Tiles per job is chosen per call: the ABI has no setter, and the test
    hooks that force a job form take it as an argument and check it on the
    host (no GPU here, so anything launched would have failed)."""
    assert not hasattr(L, "vi_set_conv_tiles_per_job")
    assert "tiles" not in open(HEADER).read()
    conv_t = L.vitest_temporal_conv_tiles
    conv_t.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 6 + [ctypes.c_void_p]
    gnconv_t = L.vitest_groupnorm_conv_tiles
    gnconv_t.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int] * 5 + [
        ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    for tiles in (0, 3, -1, 5):
        assert conv_t(A, B, Cp, D, 64, 4, 2, 64, 3, tiles, None) == INVALID
        assert gnconv_t(A, B, Cp, D, A, B, 64, 4, 2, 64, 8, 1e-5, 3, tiles, None) == INVALID
    form_t = L.vitest_temporal_attention_form
    form_t.argtypes = [ctypes.c_void_p] * 7 + [ctypes.c_int] * 9 + [ctypes.c_void_p]
    for form in (-1, 2):
        assert form_t(A, B, Cp, D, A, B, Cp, 64, 4, 2, 1, 64, 8, 8, 16, form, None) == INVALID
    assert form_t(None, None, None, None, None, None, None, 64, 4, 0, 1, 64, 8, 8, 16, 1,
                  None) == OK                                               # empty
    oproj = L.vitest_dual_attn_oproj
    oproj.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int] * 8 + [ctypes.c_void_p]
    assert oproj(A, B, Cp, D, A, B, 64, 4, 2, 6, 64, 8, 8, 16, None) == UNSUP   # C = 384
    assert oproj(A, B, Cp, D, A, B, 64, 16, 2, 1, 64, 4, 4, 16, None) == UNSUP  # L = 4
    assert oproj(A, B, Cp, D, A, B, 64, 4, 2, 1, 64, 12, 8, 16, None) == UNSUP  # context 12
    assert oproj(A, B, Cp, D, A, B, 64, 4, 2, 1, 64, 8, 8, 17, None) == UNSUP   # n_global 17
    # the forced fused form of the module refuses the same shapes before any launch
    # (seven distinct, far-apart buffers: the module checks that none overlap)
    bufs = [(i + 1) << 40 for i in range(7)]
    assert form_t(*bufs, 64, 4, 2, 1, 64, 12, 8, 16, 1, None) == UNSUP
    assert oproj(None, None, None, None, None, None, 64, 4, 0, 1, 64, 8, 8, 16, None) == OK
    assert conv_t(None, None, None, None, 64, 4, 0, 64, 3, 1, None) == OK     # empty
    assert conv_t(A, B, Cp, D, 64, 4, 2, 64, 2, 1, None) == INVALID         # even k
    assert conv_t(A + 4, B, Cp, D, 64, 4, 2, 64, 3, 2, None) == ALIGN


def test_empty_calls_succeed_without_touching_pointers(L):
    """P == 0: valid, nothing to compute; NULL pointers are fine and nothing is
    launched (no device here, so any CUDA call would have failed)."""
    n0 = vi.launch_count()
    assert attn(L, q=None, k=None, v=None, o=None, P=0) == OK
    assert attn(L, q=None, k=None, v=None, o=None, P=0, f32=True) == OK
    assert conv(L, x=None, w=None, b=None, y=None, P=0) == OK
    assert gn(L, x=None, g=None, bt=None, y=None, P=0) == OK
    assert gnconv(L, x=None, g=None, bt=None, w=None, b=None, y=None, P=0) == OK
    assert tattn(L, x=None, wqkv=None, bqkv=None, wo=None, bo=None, out=None, ws=None, P=0) == OK
    assert L.vi_groupnorm_global_noalloc(None, None, None, None, 64, 4, 0, 64, 8, 1e-5, None) == OK
    assert vi.launch_count() == n0


@pytest.mark.parametrize("call,expect", [
    (lambda L: attn(L, P=0, F=0), INVALID), (lambda L: attn(L, P=0, d=32), UNSUP),
    (lambda L: attn(L, P=0, pre=17), INVALID), (lambda L: conv(L, P=0, k=2), INVALID),
    (lambda L: gn(L, P=0, groups=7), INVALID), (lambda L: gnconv(L, P=0, N=3), INVALID),
    (lambda L: tattn(L, P=0, heads=0), INVALID),
])
def test_empty_calls_still_check_scalar_arguments(L, call, expect):
    assert call(L) == expect


def test_binding_checks_shapes_before_the_call():
    """Sizes come from the first tensor; the others must match it (a smaller
    tensor would be read out of bounds by the kernel)."""
    import torch
    from clip_temporal_modules_b200._binding import _shape
    _shape(torch.empty(2, 3, 4), (2, 3, 4), "x")
    with pytest.raises(ValueError):
        _shape(torch.empty(2, 3, 4), (2, 3, 5), "x")
    with pytest.raises(ValueError):
        _shape(torch.empty(12), (3, 4), "w")


def attn_shard(L, q=A, ke=B, ve=Cp, kg=D, vg=E, o=G, F_loc=64, N_loc=4, clip0=4, N=16, P=2,
               heads=2, d=64, pre=8, post=8, glob=16, part=0):
    return L.vi_dual_attn_shard(q, ke, ve, kg, vg, o, F_loc, N_loc, clip0, N, P, heads, d, pre,
                                post, glob, part, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(N_loc=0), INVALID), (dict(F_loc=62), INVALID), (dict(clip0=13), INVALID),
    (dict(clip0=-1), INVALID), (dict(N=3), INVALID), (dict(pre=17), INVALID),
    (dict(glob=17), UNSUP), (dict(F_loc=128), UNSUP), (dict(d=32), UNSUP), (dict(P=-1), INVALID),
    (dict(q=A + 8), ALIGN), (dict(o=A), INVALID), (dict(q=None), INVALID),
    (dict(P=0, q=None, ke=None, ve=None, kg=None, vg=None, o=None), OK),
    (dict(part=3), INVALID), (dict(part=-1), INVALID),
    (dict(P=0, q=None, ke=None, ve=None, kg=None, vg=None, o=None, part=1), OK),
])
def test_attention_shard_rejects(L, kw, expect):
    assert attn_shard(L, **kw) == expect


@pytest.mark.parametrize("kw,expect", [
    (dict(k=2), INVALID), (dict(F_loc=0), INVALID), (dict(C=40), UNSUP), (dict(x=A + 8), ALIGN),
    (dict(y=A), INVALID), (dict(P=0, x=None, w=None, b=None, y=None), OK),
    (dict(part=3), INVALID), (dict(P=0, x=None, w=None, b=None, y=None, part=2), OK),
])
def test_conv_shard_rejects(L, kw, expect):
    a = dict(x=A, w=B, b=Cp, y=D, F_loc=64, P=2, C=64, k=3, part=0)
    a.update(kw)
    assert L.vi_temporal_conv_shard(a["x"], a["w"], a["b"], a["y"], a["F_loc"], a["P"], a["C"],
                                    a["k"], a["part"], None) == expect


def test_groupnorm_shard_rejects(L):
    st = L.vi_groupnorm_shard_stats
    ap = L.vi_groupnorm_shard_apply
    assert st(A, 64, 0, 64, 8, B, None) == INVALID          # a shard with no rows has no stats
    assert st(A, 64, 2, 64, 7, B, None) == INVALID
    assert st(None, 64, 2, 64, 8, B, None) == INVALID
    assert st(A + 8, 64, 2, 64, 8, B, None) == ALIGN
    assert ap(A, B, 0, Cp, D, E, 64, 2, 64, 8, 1e-5, None) == INVALID     # W = 0
    assert ap(A, B, 2, Cp, D, E, 64, 2, 64, 8, -1.0, None) == INVALID     # eps < 0
    assert ap(A, B, 2, Cp, D, A + 64, 64, 2, 64, 8, 1e-5, None) == INVALID  # y inside x
