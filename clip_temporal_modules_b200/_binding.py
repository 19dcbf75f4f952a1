"""ctypes binding of libvi (include/vi.h): argument marshalling only.

Every step of the temporal modules runs in the CUDA kernels behind the C ABI;
this module checks that tensors are what the ABI expects (device, dtype,
contiguity, shape), passes raw pointers and the current CUDA stream, and turns
a negative status into an exception.  There is no CPU path: if libvi.so is
missing the calls raise.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libvi.so")

VI_OK = 0
STATUS = {0: "VI_OK", -1: "VI_ERR_INVALID_ARG", -2: "VI_ERR_ALIGNMENT", -3: "VI_ERR_UNSUPPORTED",
          -4: "VI_ERR_CUDA", -5: "VI_ERR_DEVICE_TIMEOUT"}

# name -> argument types (all return int status)
_vp, _i, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
SIGNATURES = {
    "vi_dual_attn": [_vp, _vp, _vp, _vp] + [_i] * 8 + [_vp],
    "vi_dual_attn_f32": [_vp, _vp, _vp, _vp] + [_i] * 8 + [_vp],
    "vi_temporal_conv": [_vp, _vp, _vp, _vp] + [_i] * 5 + [_vp],
    "vi_temporal_conv_f32": [_vp, _vp, _vp, _vp] + [_i] * 5 + [_vp],
    "vi_groupnorm_global": [_vp, _vp, _vp, _vp] + [_i] * 5 + [_f, _vp],
    "vi_groupnorm_global_f32": [_vp, _vp, _vp, _vp] + [_i] * 5 + [_f, _vp],
    "vi_groupnorm_global_noalloc": [_vp, _vp, _vp, _vp] + [_i] * 5 + [_f, _vp],
    "vi_groupnorm_conv": [_vp] * 6 + [_i] * 5 + [_f, _i, _vp],
    "vi_temporal_attention": [_vp] * 7 + [_i] * 8 + [_vp],
    "vi_selftest_wait_timeout": [_i, _vp],
    "vi_dual_attn_shard": [_vp] * 6 + [_i] * 11 + [_vp],
    "vi_temporal_conv_shard": [_vp] * 4 + [_i] * 5 + [_vp],
    "vi_groupnorm_shard_stats": [_vp] + [_i] * 4 + [_vp, _vp],
    "vi_groupnorm_shard_apply": [_vp, _vp, _i, _vp, _vp, _vp] + [_i] * 4 + [_f, _vp],
    "vi_version": [],
    "vi_take_device_errors": [],
}


class ViError(RuntimeError):
    def __init__(self, name: str, status: int):
        super().__init__(f"{name} returned {status} ({STATUS.get(status, 'unknown')})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load libvi.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libvi.so not built at {LIB_PATH}; run __graft_entry__.build()")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.vi_temporal_attention_workspace_bytes.argtypes = [_i, _i, _i]
        L.vi_temporal_attention_workspace_bytes.restype = ctypes.c_ulonglong
        L.vi_launch_count.argtypes = []
        L.vi_launch_count.restype = ctypes.c_ulonglong
        L.vi_status_string.argtypes = [ctypes.c_int]
        L.vi_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(name: str, status: int) -> None:
    if status != VI_OK:
        raise ViError(name, status)


def _stream_ptr(stream) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _suffix(t) -> str:
    import torch
    if t.dtype == torch.bfloat16:
        return ""
    if t.dtype == torch.float32:
        return "_f32"
    raise TypeError(f"libvi takes bfloat16 or float32 tensors, got {t.dtype}")


def _dev(*ts):
    for t in ts:
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("libvi takes contiguous CUDA tensors")
    if len({t.dtype for t in ts}) != 1:
        raise TypeError("all tensors of one call share a dtype")


def _shape(t, shape, what: str) -> None:
    """The C ABI takes sizes, not shapes: a tensor smaller than the sizes say
    would be read or written out of bounds, so shapes are checked here."""
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{what}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


def dual_attn(q, k, v, out=None, *, N: int, heads: int, n_pre: int = 8, n_post: int = 8,
              n_global: int = 16, stream=None):
    """Dual-domain temporal attention; q, k, v, out are [P][F][heads*d] CUDA tensors."""
    import torch
    if out is None:
        out = torch.empty_like(q)
    _dev(q, k, v, out)
    P, F, C = q.shape
    for t, n in ((k, "k"), (v, "v"), (out, "out")):
        _shape(t, q.shape, n)
    name = "vi_dual_attn" + _suffix(q)
    _check(name, getattr(lib(), name)(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                      F, N, P, heads, C // heads, n_pre, n_post, n_global,
                                      _stream_ptr(stream)))
    return out


def temporal_conv(x, w, b, out=None, *, N: int, stream=None):
    """Clip-padded temporal conv; x, out [P][F][C], w [C][C][k], b [C] CUDA tensors."""
    import torch
    if out is None:
        out = torch.empty_like(x)
    _dev(x, w, b, out)
    P, F, C = x.shape
    if w.dim() != 3:
        raise ValueError("w: expected [C_out][C_in][k]")
    k = w.shape[2]
    _shape(w, (C, C, k), "w")
    _shape(b, (C,), "b")
    _shape(out, x.shape, "out")
    name = "vi_temporal_conv" + _suffix(x)
    _check(name, getattr(lib(), name)(x.data_ptr(), w.data_ptr(), b.data_ptr(), out.data_ptr(),
                                      F, N, P, C, k, _stream_ptr(stream)))
    return out


def groupnorm_global(x, gamma, beta, out=None, *, N: int, groups: int, eps: float = 1e-5,
                     stream=None):
    """Global-statistics GroupNorm; x, out [P][F][C] (out may be x), gamma/beta [C]."""
    import torch
    if out is None:
        out = torch.empty_like(x)
    _dev(x, gamma, beta, out)
    P, F, C = x.shape
    _shape(gamma, (C,), "gamma")
    _shape(beta, (C,), "beta")
    _shape(out, x.shape, "out")
    name = "vi_groupnorm_global" + _suffix(x)
    _check(name, getattr(lib(), name)(x.data_ptr(), gamma.data_ptr(), beta.data_ptr(),
                                      out.data_ptr(), F, N, P, C, groups, float(eps),
                                      _stream_ptr(stream)))
    return out


def groupnorm_conv(x, gamma, beta, w, b, out=None, *, N: int, groups: int, eps: float = 1e-5,
                   stream=None):
    """Fused GroupNorm (global statistics) -> temporal conv; bf16 CUDA tensors."""
    import torch
    if out is None:
        out = torch.empty_like(x)
    _dev(x, gamma, beta, w, b, out)
    P, F, C = x.shape
    if w.dim() != 3:
        raise ValueError("w: expected [C_out][C_in][k]")
    _shape(w, (C, C, w.shape[2]), "w")
    for t, n in ((gamma, "gamma"), (beta, "beta"), (b, "b")):
        _shape(t, (C,), n)
    _shape(out, x.shape, "out")
    _check("vi_groupnorm_conv", lib().vi_groupnorm_conv(
        x.data_ptr(), gamma.data_ptr(), beta.data_ptr(), w.data_ptr(), b.data_ptr(),
        out.data_ptr(), F, N, P, C, groups, float(eps), w.shape[2], _stream_ptr(stream)))
    return out


def temporal_attention(x, w_qkv, b_qkv, w_out, b_out, out=None, workspace=None, *, N: int,
                       heads: int, n_pre: int = 8, n_post: int = 8, n_global: int = 16,
                       stream=None):
    """Projections + dual-domain attention + output projection; bf16 CUDA tensors.
    w_qkv [3C][C], b_qkv [3C], w_out [C][C], b_out [C] (Linear layout)."""
    import torch
    P, F, C = x.shape
    if out is None:
        out = torch.empty_like(x)
    if workspace is None:
        n = int(lib().vi_temporal_attention_workspace_bytes(F, P, C))
        workspace = torch.empty(n // 2, dtype=torch.bfloat16, device=x.device)
    _dev(x, w_qkv, b_qkv, w_out, b_out, out, workspace)
    _shape(w_qkv, (3 * C, C), "w_qkv")
    _shape(b_qkv, (3 * C,), "b_qkv")
    _shape(w_out, (C, C), "w_out")
    _shape(b_out, (C,), "b_out")
    _shape(out, x.shape, "out")
    if workspace.numel() * workspace.element_size() < 4 * P * F * C * 2:
        raise ValueError("workspace: smaller than vi_temporal_attention_workspace_bytes")
    _check("vi_temporal_attention", lib().vi_temporal_attention(
        x.data_ptr(), w_qkv.data_ptr(), b_qkv.data_ptr(), w_out.data_ptr(), b_out.data_ptr(),
        out.data_ptr(), workspace.data_ptr(), F, N, P, heads, C // heads, n_pre, n_post, n_global,
        _stream_ptr(stream)))
    return out


def dual_attn_shard(q, k_ext, v_ext, k_glob, v_glob, out=None, *, N_loc: int, clip0: int,
                    N: int, heads: int, n_pre: int = 8, n_post: int = 8, n_global: int = 16,
                    part: int = 0, stream=None):
    """Dual-domain attention of one shard of a video cut along frames (bf16).

    q, out [P][F_loc][C]; k_ext, v_ext [P][F_loc + 16][C] (halo-padded: 8
    frames before and after the shard around it); k_glob, v_glob
    [P][n_global][C]; part 0 all, 1 interior blocks, 2 boundary blocks."""
    import torch
    if out is None:
        out = torch.empty_like(q)
    if n_global == 0 and (k_glob is None or v_glob is None):
        k_glob, v_glob = k_ext, v_ext          # not read without global frames
    _dev(q, k_ext, v_ext, k_glob, v_glob, out)
    P, F_loc, C = q.shape
    _shape(out, q.shape, "out")
    _shape(k_ext, (P, F_loc + 16, C), "k_ext")
    _shape(v_ext, (P, F_loc + 16, C), "v_ext")
    if n_global > 0:
        _shape(k_glob, (P, n_global, C), "k_glob")
        _shape(v_glob, (P, n_global, C), "v_glob")
    _check("vi_dual_attn_shard", lib().vi_dual_attn_shard(
        q.data_ptr(), k_ext.data_ptr(), v_ext.data_ptr(), k_glob.data_ptr(), v_glob.data_ptr(),
        out.data_ptr(), F_loc, N_loc, clip0, N, P, heads, C // heads, n_pre, n_post, n_global,
        int(part), _stream_ptr(stream)))
    return out


def temporal_conv_shard(x_ext, w, b, out=None, *, part: int = 0, stream=None):
    """Temporal conv of one shard: x_ext [P][F_loc + 2(k/2)][C] (halo-padded)
    -> [P][F_loc][C] (bf16); part 0 all, 1 interior blocks, 2 boundary blocks."""
    import torch
    _dev(x_ext, w, b)
    if w.dim() != 3:
        raise ValueError("w: expected [C_out][C_in][k]")
    P, Fx, C = x_ext.shape
    k = w.shape[2]
    F_loc = Fx - 2 * (k // 2)
    if out is None:
        out = torch.empty((P, F_loc, C), dtype=x_ext.dtype, device=x_ext.device)
    _dev(x_ext, w, b, out)
    _shape(w, (C, C, k), "w")
    _shape(b, (C,), "b")
    _shape(out, (P, F_loc, C), "out")
    _check("vi_temporal_conv_shard", lib().vi_temporal_conv_shard(
        x_ext.data_ptr(), w.data_ptr(), b.data_ptr(), out.data_ptr(), F_loc, P, C, k, int(part),
        _stream_ptr(stream)))
    return out


def groupnorm_shard_stats(x, *, groups: int, out=None, stream=None):
    """Per-group (mean, var) of one shard's rows: a [groups][2] float64 CUDA tensor
    (`out` if given, e.g. this shard's slot of a gathered [W][groups][2] tensor)."""
    import torch
    _dev(x)
    P, F_loc, C = x.shape
    if out is None:
        stats = torch.empty((groups, 2), dtype=torch.float64, device=x.device)
    else:
        if not out.is_cuda or out.dtype != torch.float64 or tuple(out.shape) != (groups, 2) \
                or not out.is_contiguous():
            raise ValueError("out: expected a contiguous [groups][2] float64 CUDA tensor")
        stats = out
    _check("vi_groupnorm_shard_stats", lib().vi_groupnorm_shard_stats(
        x.data_ptr(), F_loc, P, C, groups, stats.data_ptr(), _stream_ptr(stream)))
    return stats


def groupnorm_shard_apply(x, shard_stats, gamma, beta, out=None, *, eps: float = 1e-5,
                          stream=None):
    """Normalise one shard with the W shards' statistics shard_stats [W][groups][2]."""
    import torch
    if out is None:
        out = torch.empty_like(x)
    _dev(x, gamma, beta, out)
    if not shard_stats.is_cuda or shard_stats.dtype != torch.float64 or shard_stats.dim() != 3 \
            or not shard_stats.is_contiguous():
        raise ValueError("shard_stats: expected a contiguous [W][groups][2] float64 CUDA tensor")
    P, F_loc, C = x.shape
    W, groups = shard_stats.shape[0], shard_stats.shape[1]
    _shape(shard_stats, (W, groups, 2), "shard_stats")
    _shape(gamma, (C,), "gamma")
    _shape(beta, (C,), "beta")
    _shape(out, x.shape, "out")
    _check("vi_groupnorm_shard_apply", lib().vi_groupnorm_shard_apply(
        x.data_ptr(), shard_stats.data_ptr(), W, gamma.data_ptr(), beta.data_ptr(),
        out.data_ptr(), F_loc, P, C, groups, float(eps), _stream_ptr(stream)))
    return out


def launch_count() -> int:
    """Kernels libvi has launched in this process so far."""
    return int(lib().vi_launch_count())


def conv_forced_tiles(x, w, b, out=None, *, N: int, tiles: int, stream=None):
    """Test hook (not part of the ABI in vi.h): the bf16 tensor-core conv with
    its tiles per job forced to 1 or 2, so that tests reach both job forms."""
    import torch
    if out is None:
        out = torch.empty_like(x)
    _dev(x, w, b, out)
    P, F, C = x.shape
    k = w.shape[2]
    _shape(w, (C, C, k), "w")
    _shape(b, (C,), "b")
    _shape(out, x.shape, "out")
    fn = lib().vitest_temporal_conv_tiles
    fn.argtypes = [_vp] * 4 + [_i] * 6 + [_vp]
    fn.restype = ctypes.c_int
    _check("vitest_temporal_conv_tiles", fn(x.data_ptr(), w.data_ptr(), b.data_ptr(),
                                            out.data_ptr(), F, N, P, C, k, int(tiles),
                                            _stream_ptr(stream)))
    return out


def groupnorm_conv_forced_tiles(x, gamma, beta, w, b, out=None, *, N: int, groups: int,
                                tiles: int, eps: float = 1e-5, stream=None):
    """Test hook (not part of the ABI in vi.h): the fused GroupNorm -> conv with
    the conv's tiles per job forced to 1 or 2."""
    import torch
    if out is None:
        out = torch.empty_like(x)
    _dev(x, gamma, beta, w, b, out)
    P, F, C = x.shape
    _shape(w, (C, C, w.shape[2]), "w")
    for t, n in ((gamma, "gamma"), (beta, "beta"), (b, "b")):
        _shape(t, (C,), n)
    _shape(out, x.shape, "out")
    fn = lib().vitest_groupnorm_conv_tiles
    fn.argtypes = [_vp] * 6 + [_i] * 5 + [_f, _i, _i, _vp]
    fn.restype = ctypes.c_int
    _check("vitest_groupnorm_conv_tiles", fn(
        x.data_ptr(), gamma.data_ptr(), beta.data_ptr(), w.data_ptr(), b.data_ptr(),
        out.data_ptr(), F, N, P, C, groups, float(eps), w.shape[2], int(tiles),
        _stream_ptr(stream)))
    return out


def temporal_attention_forced_form(x, w_qkv, b_qkv, w_out, b_out, out=None, workspace=None, *,
                                   N: int, heads: int, fused: bool, n_pre: int = 8,
                                   n_post: int = 8, n_global: int = 16, stream=None):
    """Test hook (not part of the ABI in vi.h): the attention module with its
    form forced: the output projection fused into the attention kernel
    (fused=True), or the attention kernel followed by the output GEMM."""
    import torch
    P, F, C = x.shape
    if out is None:
        out = torch.empty_like(x)
    if workspace is None:
        n = int(lib().vi_temporal_attention_workspace_bytes(F, P, C))
        workspace = torch.empty(n // 2, dtype=torch.bfloat16, device=x.device)
    _dev(x, w_qkv, b_qkv, w_out, b_out, out, workspace)
    _shape(w_qkv, (3 * C, C), "w_qkv")
    _shape(b_qkv, (3 * C,), "b_qkv")
    _shape(w_out, (C, C), "w_out")
    _shape(b_out, (C,), "b_out")
    _shape(out, x.shape, "out")
    if workspace.numel() * workspace.element_size() < 4 * P * F * C * 2:
        raise ValueError("workspace: smaller than vi_temporal_attention_workspace_bytes")
    fn = lib().vitest_temporal_attention_form
    fn.argtypes = [_vp] * 7 + [_i] * 9 + [_vp]
    fn.restype = ctypes.c_int
    _check("vitest_temporal_attention_form", fn(
        x.data_ptr(), w_qkv.data_ptr(), b_qkv.data_ptr(), w_out.data_ptr(), b_out.data_ptr(),
        out.data_ptr(), workspace.data_ptr(), F, N, P, heads, C // heads, n_pre, n_post, n_global,
        1 if fused else 0, _stream_ptr(stream)))
    return out


def dual_attn_oproj(q, k, v, w_out, b_out, out=None, *, N: int, heads: int, n_pre: int = 8,
                    n_post: int = 8, n_global: int = 16, stream=None):
    """Test hook (not part of the ABI in vi.h): the attention kernel with the
    module's output projection fused in, out = dual_attn(q, k, v) W_out^T +
    b_out; bf16 CUDA tensors, w_out [C][C] and b_out [C] in the Linear layout."""
    import torch
    if out is None:
        out = torch.empty_like(q)
    _dev(q, k, v, w_out, b_out, out)
    P, F, C = q.shape
    for t, n in ((k, "k"), (v, "v"), (out, "out")):
        _shape(t, q.shape, n)
    _shape(w_out, (C, C), "w_out")
    _shape(b_out, (C,), "b_out")
    fn = lib().vitest_dual_attn_oproj
    fn.argtypes = [_vp] * 6 + [_i] * 8 + [_vp]
    fn.restype = ctypes.c_int
    _check("vitest_dual_attn_oproj", fn(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), w_out.data_ptr(), b_out.data_ptr(),
        out.data_ptr(), F, N, P, heads, C // heads, n_pre, n_post, n_global,
        _stream_ptr(stream)))
    return out


def take_device_errors() -> None:
    """Synchronise and raise if a kernel's bounded wait ran out since the last call."""
    _check("vi_take_device_errors", lib().vi_take_device_errors())
