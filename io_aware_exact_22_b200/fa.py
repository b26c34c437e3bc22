"""ctypes binding over libfa.so (C ABI in include/fa.h).

Every name in ``EXPORTS`` (``fa_fwd``, ``fa_bwd``, the split-KV, FP8, deterministic,
allocation-free and sharded-pieces entry points, the status and self-test calls) has a
function here with the C name that only marshals arguments: torch tensors supply device
pointers and the current CUDA stream, and every step of the attention path runs in the
library's kernels.  ``forward``, ``forward_splitkv``, ``forward_fp8`` and ``backward``
additionally allocate the output tensors with torch (memory plumbing only).

Loading fails loudly (``RuntimeError``) when the shared library is missing: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("FA_LIB_PATH", os.path.join(_HERE, "libfa.so"))

STATUS = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_CUDA",
          4: "FA_ERR_TIMEOUT", 5: "FA_ERR_DEVICE_CHECK"}
EXPORTS = ("fa_fwd", "fa_bwd", "fa_bwd_workspace_bytes", "fa_get_device_status",
           "fa_status_string", "fa_version", "fa_bwd_noalloc", "fa_selftest_wait_timeout",
           "fa_fwd_splitkv", "fa_fwd_splitkv_workspace_bytes", "fa_fwd_splitkv_default_splits",
           "fa_bwd_deterministic", "fa_fwd_fp8", "fa_fwd_partial", "fa_merge_partials", "fa_fwd_carry",
           "fa_bwd_prepare", "fa_bwd_accumulate", "fa_bwd_finish", "fa_bwd_contribute", "fa_bwd_acc_add",
           "fa_bwd_main", "fa_bwd_dq_post",
           "fa_debug_build", "fa_debug_visits")
# Size of the library's built-in scratch used by fa_bwd_noalloc (include/fa.h).
NOALLOC_MAX_SCRATCH_BYTES = 64 << 20

_lib = None


class FAError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what} failed: {STATUS.get(code, code)}")
        self.code = code


def lib() -> ctypes.CDLL:
    """Load libfa.so once; raise RuntimeError if it is not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libfa.so not found at {LIB_PATH}; build it with "
                               "`python -m io_aware_exact_22_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
        L.fa_fwd.restype = i
        L.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
        L.fa_fwd_fp8.restype = i
        L.fa_fwd_partial.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
        L.fa_fwd_partial.restype = i
        L.fa_merge_partials.argtypes = [vp, vp, i, vp, vp, i, i, i, i, vp]
        L.fa_merge_partials.restype = i
        L.fa_fwd_carry.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp]
        L.fa_fwd_carry.restype = i
        L.fa_bwd_prepare.argtypes = [vp, vp, vp, vp, sz, i, i, i, i, vp]
        L.fa_bwd_prepare.restype = i
        L.fa_bwd_accumulate.argtypes = [vp, vp, vp, vp, vp, sz, vp, vp, i, i, i, i, f, i, vp]
        L.fa_bwd_accumulate.restype = i
        L.fa_bwd_finish.argtypes = [vp, sz, vp, vp, vp, vp, vp, i, i, i, i, f, vp]
        L.fa_bwd_finish.restype = i
        L.fa_bwd_contribute.argtypes = [vp, vp, vp, vp, vp, sz, vp, vp, i, i, i, i, f, i, vp]
        L.fa_bwd_contribute.restype = i
        L.fa_bwd_acc_add.argtypes = [vp, vp, i, i, i, i, vp]
        L.fa_bwd_acc_add.restype = i
        L.fa_bwd_main.argtypes = [vp, vp, vp, vp, vp, sz, vp, vp, i, i, i, i, f, i, vp]
        L.fa_bwd_main.restype = i
        L.fa_bwd_dq_post.argtypes = [vp, sz, vp, i, i, i, i, f, vp]
        L.fa_bwd_dq_post.restype = i
        L.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, f, i, vp]
        L.fa_bwd.restype = i
        L.fa_bwd_workspace_bytes.argtypes = [i, i, i, i]
        L.fa_bwd_workspace_bytes.restype = sz
        L.fa_get_device_status.argtypes = [vp]
        L.fa_get_device_status.restype = i
        L.fa_status_string.argtypes = [i]
        L.fa_status_string.restype = ctypes.c_char_p
        L.fa_version.argtypes = []
        L.fa_version.restype = i
        L.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
        L.fa_bwd_noalloc.restype = i
        L.fa_selftest_wait_timeout.argtypes = [i, vp]
        L.fa_selftest_wait_timeout.restype = i
        L.fa_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp, sz, vp]
        L.fa_fwd_splitkv.restype = i
        L.fa_fwd_splitkv_workspace_bytes.argtypes = [i, i, i, i, i]
        L.fa_fwd_splitkv_workspace_bytes.restype = sz
        L.fa_fwd_splitkv_default_splits.argtypes = [i, i, i, i, i]
        L.fa_fwd_splitkv_default_splits.restype = i
        L.fa_debug_build.argtypes = []
        L.fa_debug_build.restype = i
        L.fa_debug_visits.argtypes = [vp, sz, i, vp]
        L.fa_debug_visits.restype = i
        L.fa_bwd_deterministic.argtypes = L.fa_bwd.argtypes
        L.fa_bwd_deterministic.restype = i
        _lib = L
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ------------------------------------------------------------------ C-named wrappers
def fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, stream=None) -> int:
    return lib().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                        float(scale), int(causal), _stream(stream))


def fa_fwd_fp8(q, k, v, descale_q, descale_k, descale_v, o, lse, B, H, N, d, scale, causal,
               stream=None) -> int:
    return lib().fa_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(descale_q), _ptr(descale_k),
                            _ptr(descale_v), _ptr(o), _ptr(lse), B, H, N, d, float(scale),
                            int(causal), _stream(stream))


def fa_fwd_partial(q, k, v, o_part, lse_part, B, H, N, d, scale, causal, stream=None) -> int:
    return lib().fa_fwd_partial(_ptr(q), _ptr(k), _ptr(v), _ptr(o_part), _ptr(lse_part), B, H, N, d,
                                float(scale), int(causal), _stream(stream))


FA_CARRY_IN, FA_CARRY_FINAL = 1, 2


def fa_fwd_carry(q, k, v, o_part, lse_part, o, lse, B, H, N, d, scale, causal, flags, stream=None) -> int:
    return lib().fa_fwd_carry(_ptr(q), _ptr(k), _ptr(v), _ptr(o_part), _ptr(lse_part), _ptr(o), _ptr(lse), B, H,
                              N, d, float(scale), int(causal), int(flags), _stream(stream))


def fa_merge_partials(o_parts, lse_parts, nparts, o, lse, B, H, N, d, stream=None) -> int:
    return lib().fa_merge_partials(_ptr(o_parts), _ptr(lse_parts), int(nparts), _ptr(o), _ptr(lse), B, H,
                                   N, d, _stream(stream))


def fa_bwd_prepare(o, dO, lse, workspace, workspace_bytes, B, H, N, d, stream=None) -> int:
    return lib().fa_bwd_prepare(_ptr(o), _ptr(dO), _ptr(lse), _ptr(workspace), int(workspace_bytes), B, H,
                                N, d, _stream(stream))


def fa_bwd_accumulate(q, k, v, dO, workspace, workspace_bytes, dk_acc, dv_acc, B, H, N, d, scale,
                      causal, stream=None) -> int:
    return lib().fa_bwd_accumulate(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(workspace),
                                   int(workspace_bytes), _ptr(dk_acc), _ptr(dv_acc), B, H, N, d,
                                   float(scale), int(causal), _stream(stream))


def fa_bwd_finish(workspace, workspace_bytes, dk_acc, dv_acc, dq, dk, dv, B, H, N, d, scale,
                  stream=None) -> int:
    return lib().fa_bwd_finish(_ptr(workspace), int(workspace_bytes), _ptr(dk_acc), _ptr(dv_acc),
                               _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, float(scale), _stream(stream))


def fa_bwd_contribute(q, k, v, dO, workspace, workspace_bytes, dk_out, dv_out, B, H, N, d, scale, causal,
                      stream=None) -> int:
    return lib().fa_bwd_contribute(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(workspace), int(workspace_bytes),
                                   _ptr(dk_out), _ptr(dv_out), B, H, N, d, float(scale), int(causal),
                                   _stream(stream))


def fa_bwd_acc_add(acc, x, B, H, N, d, stream=None) -> int:
    return lib().fa_bwd_acc_add(_ptr(acc), _ptr(x), B, H, N, d, _stream(stream))


def fa_bwd_main(q, k, v, dO, workspace, workspace_bytes, dk, dv, B, H, N, d, scale, causal,
                stream=None) -> int:
    return lib().fa_bwd_main(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(workspace), int(workspace_bytes),
                             _ptr(dk), _ptr(dv), B, H, N, d, float(scale), int(causal), _stream(stream))


def fa_bwd_dq_post(workspace, workspace_bytes, dq, B, H, N, d, scale, stream=None) -> int:
    return lib().fa_bwd_dq_post(_ptr(workspace), int(workspace_bytes), _ptr(dq), B, H, N, d, float(scale),
                                _stream(stream))


def fa_fwd_splitkv(q, k, v, o, lse, B, H, N, d, scale, causal, num_splits, workspace,
                   workspace_bytes, stream=None) -> int:
    return lib().fa_fwd_splitkv(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                                float(scale), int(causal), int(num_splits), _ptr(workspace),
                                int(workspace_bytes), _stream(stream))


def fa_fwd_splitkv_workspace_bytes(B, H, N, d, num_splits) -> int:
    return lib().fa_fwd_splitkv_workspace_bytes(B, H, N, d, num_splits)


def fa_fwd_splitkv_default_splits(B, H, N, d, causal) -> int:
    return lib().fa_fwd_splitkv_default_splits(B, H, N, d, int(causal))


def fa_bwd(q, k, v, o, dO, lse, dq, dk, dv, workspace, workspace_bytes, B, H, N, d, scale,
           causal, stream=None) -> int:
    return lib().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse), _ptr(dq),
                        _ptr(dk), _ptr(dv), _ptr(workspace), int(workspace_bytes), B, H, N, d,
                        float(scale), int(causal), _stream(stream))


def fa_bwd_deterministic(q, k, v, o, dO, lse, dq, dk, dv, workspace, workspace_bytes, B, H, N, d,
                         scale, causal, stream=None) -> int:
    return lib().fa_bwd_deterministic(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse),
                                      _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                                      int(workspace_bytes), B, H, N, d, float(scale), int(causal),
                                      _stream(stream))


def fa_bwd_noalloc(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal,
                   stream=None) -> int:
    """fa_bwd without a workspace: the library's fixed scratch array is used instead, for
    callers that cannot allocate device memory.  Overlapping calls race on that array."""
    return lib().fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dO), _ptr(lse),
                                _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, float(scale),
                                int(causal), _stream(stream))


def fa_bwd_workspace_bytes(B, H, N, d) -> int:
    return lib().fa_bwd_workspace_bytes(B, H, N, d)


def fa_get_device_status(stream=None) -> int:
    return lib().fa_get_device_status(_stream(stream))


def fa_selftest_wait_timeout(limit_ms: int, stream=None) -> int:
    return lib().fa_selftest_wait_timeout(int(limit_ms), _stream(stream))


def fa_status_string(code: int) -> str:
    return lib().fa_status_string(code).decode()


def fa_version() -> int:
    return lib().fa_version()


def fa_debug_build() -> int:
    return lib().fa_debug_build()


def fa_debug_visits(counts, n: int, clear: bool, stream=None) -> int:
    """Copies the first n visit counters of the debug build into `counts` (a contiguous CPU
    int32 tensor or numpy array), then zeroes them all when `clear`."""
    ptr = counts.ctypes.data if hasattr(counts, "ctypes") else _ptr(counts)
    return lib().fa_debug_visits(ptr, int(n), int(clear), _stream(stream))


# ------------------------------------------------------------------ tensor conveniences
def _check(t, name):
    if not (t.is_cuda and t.dtype == torch.bfloat16 and t.dim() == 4 and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor [B,H,N,d]")


def forward(q, k, v, causal: bool, scale: float | None = None, out=None, lse=None):
    """O, LSE = attention(q, k, v) through fa_fwd.  Inputs: contiguous bf16 [B,H,N,d] on CUDA."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n)
    B, H, N, d = q.shape
    scale = d ** -0.5 if scale is None else scale
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
    rc = fa_fwd(q, k, v, out, lse, B, H, N, d, scale, causal)
    if rc:
        raise FAError(rc, "fa_fwd")
    return out, lse


def forward_fp8(q8, k8, v8, descale_q, descale_k, descale_v, causal: bool,
                scale: float | None = None, out=None, lse=None):
    """O (bf16), LSE = attention of FP8 inputs through fa_fwd_fp8.  q8, k8, v8: contiguous
    CUDA tensors [B,H,N,d] of E4M3 codes (torch.uint8 or torch.float8_e4m3fn); descale_*:
    fp32 CUDA tensors with B*H elements, or None for 1."""
    for t, n in ((q8, "q8"), (k8, "k8"), (v8, "v8")):
        if not (t.is_cuda and t.element_size() == 1 and t.dim() == 4 and t.is_contiguous()):
            raise ValueError(f"{n} must be a contiguous CUDA tensor of E4M3 codes [B,H,N,d]")
    B, H, N, d = q8.shape
    for t, n in ((descale_q, "descale_q"), (descale_k, "descale_k"), (descale_v, "descale_v")):
        if t is not None and not (t.is_cuda and t.dtype == torch.float32 and t.numel() == B * H
                                  and t.is_contiguous()):
            raise ValueError(f"{n} must be a contiguous CUDA fp32 tensor of B*H elements")
    scale = d ** -0.5 if scale is None else scale
    if out is None:
        out = torch.empty((B, H, N, d), device=q8.device, dtype=torch.bfloat16)
    if lse is None:
        lse = torch.empty((B, H, N), device=q8.device, dtype=torch.float32)
    rc = fa_fwd_fp8(q8, k8, v8, descale_q, descale_k, descale_v, out, lse, B, H, N, d, scale,
                    causal)
    if rc:
        raise FAError(rc, "fa_fwd_fp8")
    return out, lse


def forward_splitkv(q, k, v, causal: bool, scale: float | None = None, num_splits: int = 0,
                    out=None, lse=None, workspace=None):
    """Split-KV forward (fa_fwd_splitkv); the workspace is allocated with torch if not given."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n)
    B, H, N, d = q.shape
    scale = d ** -0.5 if scale is None else scale
    sp = num_splits if num_splits > 0 else fa_fwd_splitkv_default_splits(B, H, N, d, causal)
    sp = max(1, min(sp, (N + 127) // 128))
    nbytes = fa_fwd_splitkv_workspace_bytes(B, H, N, d, sp)
    if workspace is None and nbytes > 0:
        workspace = torch.empty(nbytes, device=q.device, dtype=torch.uint8)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
    rc = fa_fwd_splitkv(q, k, v, out, lse, B, H, N, d, scale, causal, sp, workspace,
                        0 if workspace is None else workspace.numel())
    if rc:
        raise FAError(rc, "fa_fwd_splitkv")
    return out, lse


def backward(q, k, v, o, do, lse, causal: bool, scale: float | None = None, workspace=None,
             dq=None, dk=None, dv=None, deterministic: bool = False):
    """dQ, dK, dV through fa_bwd, or fa_bwd_deterministic (workspace allocated with torch when
    not given)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (do, "dO")):
        _check(t, n)
    B, H, N, d = q.shape
    scale = d ** -0.5 if scale is None else scale
    nbytes = fa_bwd_workspace_bytes(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 256), device=q.device, dtype=torch.uint8)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    fn = fa_bwd_deterministic if deterministic else fa_bwd
    rc = fn(q, k, v, o, do, lse, dq, dk, dv, workspace, workspace.numel(), B, H, N, d, scale, causal)
    if rc:
        raise FAError(rc, fn.__name__)
    return dq, dk, dv
