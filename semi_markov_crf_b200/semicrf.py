"""Thin Python binding of the C ABI in ``include/semicrf.h``.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libsemicrf_b200.so``.  PyTorch supplies device memory (tensors,
the workspace) and the current CUDA stream.  There is no CPU fallback: if the
library is missing or no CUDA device is present, the calls raise.
"""

from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["workspace_bytes", "workspace_itemize", "WS_GROUPS", "launch_shape", "prefix_center", "forward", "backward", "viterbi", "path_score",
           "get_status", "FLAG_NEGATE_GRAD",
           "strerror", "SemiCRFError", "library_path", "Workspace", "FLAG_NO_CENTER",
           "FLAG_FORWARD_ONLY", "FLAG_LOG_DOMAIN", "selftest_bounded_wait", "selftest_bounds", "ring_domains", "profile_enable", "profile_read",
           "forward_noalloc", "NOALLOC_SCRATCH_BYTES",
           "KERNELS", "lib"]

# every kernel the library launches (names used by the profiler)
KERNELS = ("prefix_reduce_kernel", "prefix_scan_kernel", "chain_exp_kernel", "chain_kernel",
           "cut_grid_kernel", "posterior_kernel", "segment_kernel",
           "finalize_positions_kernel",
           "reduce_partials_kernel", "viterbi_kernel", "viterbi_pipe_kernel", "viterbi_argmax_kernel",
           "viterbi_words_kernel", "viterbi_walk_kernel", "path_terms_kernel", "path_grad_kernel",
           "proj_grad_kernel")

FLAG_NO_CENTER = 0x1
FLAG_FORWARD_ONLY = 0x2
FLAG_LOG_DOMAIN = 0x4
FLAG_NEGATE_GRAD = 0x8
NOALLOC_SCRATCH_BYTES = 32 << 20  # SEMICRF_NOALLOC_SCRATCH_BYTES

# SEMICRF_LIBRARY=check loads the bounds-checking debug build instead
_LIBNAME = ("libsemicrf_b200_check.so" if os.environ.get("SEMICRF_LIBRARY") == "check"
            else "libsemicrf_b200.so")
library_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), _LIBNAME)
if not os.path.exists(library_path):
    raise ImportError(f"{library_path} is missing: build it with `python -m semi_markov_crf_b200.build`")

lib = ctypes.CDLL(library_path)

_vp = ctypes.c_void_p
_i = ctypes.c_int
_u = ctypes.c_uint
_sz = ctypes.c_size_t

lib.semicrf_workspace_bytes.argtypes = [_i, _i, _i, _i, _u, ctypes.POINTER(_sz)]
lib.semicrf_workspace_itemize.argtypes = [_i, _i, _i, _i, _u, ctypes.POINTER(_sz), _i]
lib.semicrf_launch_shape.argtypes = [_i, _i, _i, _i, ctypes.POINTER(ctypes.c_int32), _i]
lib.semicrf_prefix_center.argtypes = [_vp, _vp, _i, _i, _i, _u, _vp, _sz, _vp, _vp, _vp]
lib.semicrf_forward.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _u, _vp, _sz, _vp, _vp]
lib.semicrf_backward.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _u, _vp, _sz, _vp, _vp, _vp, _vp,
                                 _vp, _vp, _vp, _vp]
lib.semicrf_backward_segments.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _u, _vp, _sz, _vp, _vp,
                                          _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.semicrf_viterbi.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _u, _vp, _sz, _vp, _vp, _vp,
                                _vp]
lib.semicrf_path_score.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _u, _vp, _sz,
                                   _vp, _vp, _vp, _vp, _vp, _vp]
lib.semicrf_forward_proj.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _u, _vp, _sz,
                                     _vp, _vp]
lib.semicrf_backward_proj.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _u, _vp, _sz, _vp, _vp, _vp,
                                      _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.semicrf_viterbi_proj.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _u, _vp, _sz,
                                     _vp, _vp, _vp, _vp]
lib.semicrf_path_score_proj.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _u,
                                        _vp, _sz, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.semicrf_get_status.argtypes = [_vp, _vp, ctypes.POINTER(_i)]
lib.semicrf_strerror.argtypes = [_i]
lib.semicrf_strerror.restype = ctypes.c_char_p
lib.semicrf_source_digest.argtypes = []
lib.semicrf_source_digest.restype = ctypes.c_char_p
lib.semicrf_selftest_bounded_wait.argtypes = [_vp, _sz, _i, _vp]
lib.semicrf_selftest_bounds.argtypes = [_vp, _sz, _vp]
lib.semicrf_forward_noalloc.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _u, _vp, _vp]
lib.semicrf_ring_domains.argtypes = [_vp, _sz, _i, _i, _i, _i, _u, _vp, ctypes.POINTER(ctypes.c_int32)]
lib.semicrf_profile_enable.argtypes = [_i]
lib.semicrf_profile_read.argtypes = [ctypes.c_char_p, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_i)]
for _f in ("semicrf_backward_segments", "semicrf_launch_shape", "semicrf_workspace_itemize", "semicrf_forward_noalloc", "semicrf_profile_enable", "semicrf_profile_read", "semicrf_workspace_bytes", "semicrf_prefix_center", "semicrf_forward",
           "semicrf_backward", "semicrf_viterbi", "semicrf_path_score", "semicrf_get_status",
           "semicrf_forward_proj", "semicrf_backward_proj", "semicrf_viterbi_proj",
           "semicrf_path_score_proj",
           "semicrf_selftest_bounded_wait", "semicrf_selftest_bounds", "semicrf_ring_domains"):
    getattr(lib, _f).restype = _i


class SemiCRFError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {strerror(code)} (status {code})")


def strerror(code: int) -> str:
    return lib.semicrf_strerror(int(code)).decode()


def source_digest() -> str:
    """sha256 of the kernel sources the loaded library was built from."""
    return lib.semicrf_source_digest().decode()


def _check(rc: int, where: str):
    if rc != 0:
        if rc == 4:  # surface the CUDA runtime's own message
            try:
                torch.cuda.synchronize()
            except RuntimeError as e:
                raise SemiCRFError(rc, where) from e
        raise SemiCRFError(rc, where)


def workspace_bytes(B: int, T: int, C: int, K: int, flags: int = 0) -> int:
    n = _sz(0)
    _check(lib.semicrf_workspace_bytes(B, T, C, K, flags, ctypes.byref(n)), "semicrf_workspace_bytes")
    return int(n.value)


# workspace groups of semicrf_workspace_itemize, in the header's order
WS_GROUPS = ("other", "prefix_sums", "checkpoints", "recompute", "viterbi", "kept_rows",
             "path_score", "projections")


def workspace_itemize(B: int, T: int, C: int, K: int, flags: int = 0) -> dict:
    """Bytes of each workspace group (names of WS_GROUPS); they add up to
    :func:`workspace_bytes`."""
    arr = (_sz * len(WS_GROUPS))()
    _check(lib.semicrf_workspace_itemize(B, T, C, K, flags, arr, len(WS_GROUPS)),
           "semicrf_workspace_itemize")
    return {name: int(arr[i]) for i, name in enumerate(WS_GROUPS)}


SHAPE_FIELDS = ("ring_ctas", "labels_per_cta", "combine_lanes", "combine_weights",
                "helper_lanes", "helper_durations", "ring_threads", "delta", "n_checkpoints",
                "posterior_tile_rows", "log_durations_per_lane", "log_lanes_per_label",
                "log_labels_per_lane", "log_threads", "posterior_halo_rows", "cut_grid_spacing")


def launch_shape(B: int, T: int, C: int, K: int) -> dict:
    """The launch geometry the library picks for these sizes (diagnostic)."""
    arr = (ctypes.c_int32 * len(SHAPE_FIELDS))()
    _check(lib.semicrf_launch_shape(B, T, C, K, arr, len(SHAPE_FIELDS)), "semicrf_launch_shape")
    return {name: int(arr[i]) for i, name in enumerate(SHAPE_FIELDS)}


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need(t, dtype, name, device):
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or not t.is_cuda or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous CUDA {dtype} tensor")
    if t.device != device:
        raise TypeError(f"{name} is on {t.device}, expected {device}")
    return t


class Workspace:
    """Device workspace of the right size for (B, T, C, K, flags), allocated by torch."""

    def __init__(self, B: int, T: int, C: int, K: int, flags: int = 0, device=None):
        self.dims = (B, T, C, K)
        self.flags = flags
        self.nbytes = workspace_bytes(B, T, C, K, flags)
        self.buf = torch.empty(max(self.nbytes, 256), dtype=torch.uint8, device=device or "cuda")
        self.proj = False  # the last forward on it had boundary projections

    def matches(self, B, T, C, K, flags) -> bool:
        return self.dims == (B, T, C, K) and self.flags == flags

    @property
    def ptr(self) -> int:
        return self.buf.data_ptr()


def _projections(p_start, p_end, shape, device):
    for name, t in (("p_start", p_start), ("p_end", p_end)):
        if t is not None:
            _need(t, torch.float32, name, device)
            if tuple(t.shape) != tuple(shape):
                raise TypeError(f"{name} must have shape {tuple(shape)}")
    return p_start is not None or p_end is not None


def _flags(center: bool, forward_only: bool = False, log_domain: bool = False) -> int:
    return ((0 if center else FLAG_NO_CENTER) | (FLAG_FORWARD_ONLY if forward_only else 0) |
            (FLAG_LOG_DOMAIN if log_domain else 0))


def prefix_center(em, lengths, center: bool = True, ws: Workspace | None = None):
    """Step 1: float64 prefix sums S [B, T+1, C] and nu [B, C] (float32)."""
    dev = em.device
    _need(em, torch.float32, "em", dev)
    _need(lengths, torch.int32, "lengths", dev)
    B, T, C = em.shape
    flags = _flags(center)
    if ws is None or not ws.matches(B, T, C, 1, flags):
        ws = Workspace(B, T, C, 1, flags, dev)
    S = torch.empty((B, T + 1, C), dtype=torch.float64, device=dev)
    nu = torch.empty((B, C), dtype=torch.float32, device=dev)
    _check(lib.semicrf_prefix_center(_ptr(em), _ptr(lengths), B, T, C, flags, ws.ptr, ws.nbytes,
                                     _ptr(S), _ptr(nu), _stream(dev)), "semicrf_prefix_center")
    return S, nu


def forward(em, lengths, trans, dur, center: bool = True, forward_only: bool = False,
            ws: Workspace | None = None, logZ=None, log_domain: bool = False,
            p_start=None, p_end=None):
    """Steps 1-2: log Z [B] (float64).  Returns (logZ, workspace); pass the
    workspace to :func:`backward`.  log_domain=True runs every sequence's
    rings in the log domain (SEMICRF_FLAG_LOG_DOMAIN).  ``p_start`` /
    ``p_end`` [B,T,C] float32 are boundary projection scores
    (semicrf_forward_proj)."""
    dev = em.device
    _need(em, torch.float32, "em", dev)
    _need(lengths, torch.int32, "lengths", dev)
    _need(trans, torch.float32, "trans", dev)
    _need(dur, torch.float32, "dur", dev)
    B, T, C = em.shape
    K = dur.shape[0]
    flags = _flags(center, forward_only, log_domain)
    if ws is None or not ws.matches(B, T, C, K, flags):
        ws = Workspace(B, T, C, K, flags, dev)
    if logZ is None:
        logZ = torch.empty(B, dtype=torch.float64, device=dev)
    if _projections(p_start, p_end, (B, T, C), dev):
        _check(lib.semicrf_forward_proj(_ptr(em), _ptr(lengths), _ptr(trans), _ptr(dur),
                                        _ptr(p_start), _ptr(p_end), B, T, C, K, flags, ws.ptr,
                                        ws.nbytes, _ptr(logZ), _stream(dev)), "semicrf_forward_proj")
        ws.proj = True
    else:
        _check(lib.semicrf_forward(_ptr(em), _ptr(lengths), _ptr(trans), _ptr(dur), B, T, C, K,
                                   flags, ws.ptr, ws.nbytes, _ptr(logZ), _stream(dev)),
               "semicrf_forward")
        ws.proj = False
    return logZ, ws


def backward(ws: Workspace, lengths, trans, dur, grad_logZ=None, marginals: bool = False,
             out: dict | None = None, segments: bool = False):
    """Step 3 on the workspace of the preceding :func:`forward`.

    Returns a dict with grad_em [B,T,C], grad_trans [C,C], grad_dur [K,C]
    (float32) and, when ``marginals``, pos_marg [B,T,C], start_marg and
    end_marg [B,T+1,C]; after a forward with boundary projections also
    grad_p_start and grad_p_end [B,T,C] (semicrf_backward_proj).  With
    ``segments`` also seg_marg [B,T,K,C], P(segment [s, s+k) with label c)
    at [b, s, k-1, c] (semicrf_backward_segments; not after a forward with
    projections).  ``out`` may supply preallocated tensors."""
    B, T, C, K = ws.dims
    dev = ws.buf.device
    _need(lengths, torch.int32, "lengths", dev)
    _need(trans, torch.float32, "trans", dev)
    _need(dur, torch.float32, "dur", dev)
    if grad_logZ is not None:
        _need(grad_logZ, torch.float64, "grad_logZ", dev)
    o = {} if out is None else out
    if "grad_em" not in o:
        o["grad_em"] = torch.empty((B, T, C), dtype=torch.float32, device=dev)
        o["grad_trans"] = torch.empty((C, C), dtype=torch.float32, device=dev)
        o["grad_dur"] = torch.empty((K, C), dtype=torch.float32, device=dev)
    if marginals and "pos_marg" not in o:
        o["pos_marg"] = torch.empty((B, T, C), dtype=torch.float32, device=dev)
        o["start_marg"] = torch.empty((B, T + 1, C), dtype=torch.float32, device=dev)
        o["end_marg"] = torch.empty((B, T + 1, C), dtype=torch.float32, device=dev)
    if ws.proj:
        for name in ("grad_p_start", "grad_p_end"):
            if name not in o:
                o[name] = torch.empty((B, T, C), dtype=torch.float32, device=dev)
        _check(lib.semicrf_backward_proj(
            _ptr(lengths), _ptr(trans), _ptr(dur), B, T, C, K, ws.flags, ws.ptr, ws.nbytes,
            _ptr(grad_logZ), _ptr(o["grad_em"]), _ptr(o["grad_trans"]), _ptr(o["grad_dur"]),
            _ptr(o["grad_p_start"]), _ptr(o["grad_p_end"]),
            _ptr(o.get("pos_marg") if marginals else None),
            _ptr(o.get("start_marg") if marginals else None),
            _ptr(o.get("end_marg") if marginals else None), _stream(dev)), "semicrf_backward_proj")
        return o
    if segments:
        if ws.proj:
            raise ValueError("segment marginals are not available after a forward with projections")
        if "seg_marg" not in o:
            o["seg_marg"] = torch.empty((B, T, K, C), dtype=torch.float32, device=dev)
        _check(lib.semicrf_backward_segments(
            _ptr(lengths), _ptr(trans), _ptr(dur), B, T, C, K, ws.flags, ws.ptr, ws.nbytes,
            _ptr(grad_logZ), _ptr(o["grad_em"]), _ptr(o["grad_trans"]), _ptr(o["grad_dur"]),
            _ptr(o.get("pos_marg") if marginals else None),
            _ptr(o.get("start_marg") if marginals else None),
            _ptr(o.get("end_marg") if marginals else None), _ptr(o["seg_marg"]), _stream(dev)),
            "semicrf_backward_segments")
        return o
    _check(lib.semicrf_backward(_ptr(lengths), _ptr(trans), _ptr(dur), B, T, C, K, ws.flags, ws.ptr,
                                ws.nbytes, _ptr(grad_logZ), _ptr(o["grad_em"]), _ptr(o["grad_trans"]),
                                _ptr(o["grad_dur"]), _ptr(o.get("pos_marg") if marginals else None),
                                _ptr(o.get("start_marg") if marginals else None),
                                _ptr(o.get("end_marg") if marginals else None), _stream(dev)),
           "semicrf_backward")
    return o


def viterbi(em, lengths, trans, dur, center: bool = True, ws: Workspace | None = None,
            out=None, p_start=None, p_end=None):
    """Step 4: (score [B] float64, labels [B,T] int32, seg_start [B,T] uint8).
    ``out`` may supply that triple preallocated; ``p_start`` / ``p_end``
    [B,T,C] are boundary projection scores (semicrf_viterbi_proj)."""
    dev = em.device
    _need(em, torch.float32, "em", dev)
    _need(lengths, torch.int32, "lengths", dev)
    _need(trans, torch.float32, "trans", dev)
    _need(dur, torch.float32, "dur", dev)
    B, T, C = em.shape
    K = dur.shape[0]
    flags = _flags(center)
    if ws is None or not ws.matches(B, T, C, K, flags):
        ws = Workspace(B, T, C, K, flags, dev)
    if out is None:
        score = torch.empty(B, dtype=torch.float64, device=dev)
        labels = torch.empty((B, T), dtype=torch.int32, device=dev)
        seg = torch.empty((B, T), dtype=torch.uint8, device=dev)
    else:
        score, labels, seg = out
        _need(score, torch.float64, "score", dev)
        _need(labels, torch.int32, "labels", dev)
        _need(seg, torch.uint8, "seg_start", dev)
    if _projections(p_start, p_end, (B, T, C), dev):
        _check(lib.semicrf_viterbi_proj(_ptr(em), _ptr(lengths), _ptr(trans), _ptr(dur),
                                        _ptr(p_start), _ptr(p_end), B, T, C, K, flags, ws.ptr,
                                        ws.nbytes, _ptr(score), _ptr(labels), _ptr(seg),
                                        _stream(dev)), "semicrf_viterbi_proj")
        ws.proj = True
        return score, labels, seg
    _check(lib.semicrf_viterbi(_ptr(em), _ptr(lengths), _ptr(trans), _ptr(dur), B, T, C, K, flags,
                               ws.ptr, ws.nbytes, _ptr(score), _ptr(labels), _ptr(seg), _stream(dev)),
           "semicrf_viterbi")
    ws.proj = False
    return score, labels, seg


def path_score(em, lengths, trans, dur, labels, seg_start, center: bool = True,
               ws: Workspace | None = None, grad_score=None, negate: bool = False,
               grads: dict | None = None, score=None, p_start=None, p_end=None):
    """Score [B] (float64) of given segmentations, NaN where malformed.

    ``labels`` [B,T] int32 and ``seg_start`` [B,T] uint8 as :func:`viterbi`
    returns them.  ``grads`` may hold any of grad_em [B,T,C], grad_trans
    [C,C], grad_dur [K,C] (float32): w_b * d score_b / d x is ADDED into
    them, w_b = grad_score[b] (float64 [B], None = ones), negated when
    ``negate``.  For the NLL log Z - score: :func:`backward` with grad_logZ=g,
    then this call with grad_score=g, negate=True and the same dict.  ``ws``
    may be the workspace of a :func:`forward` with the same sizes (the path
    score has a region of its own).  ``p_start`` / ``p_end`` [B,T,C] add the
    boundary projection terms (semicrf_path_score_proj), and ``grads`` may
    then also hold grad_p_start / grad_p_end [B,T,C]."""
    dev = em.device
    _need(em, torch.float32, "em", dev)
    _need(lengths, torch.int32, "lengths", dev)
    _need(trans, torch.float32, "trans", dev)
    _need(dur, torch.float32, "dur", dev)
    _need(labels, torch.int32, "labels", dev)
    _need(seg_start, torch.uint8, "seg_start", dev)
    B, T, C = em.shape
    K = dur.shape[0]
    flags = _flags(center) | (FLAG_NEGATE_GRAD if negate else 0)
    if ws is None or ws.dims != (B, T, C, K):
        ws = Workspace(B, T, C, K, _flags(center), dev)
    if grad_score is not None:
        _need(grad_score, torch.float64, "grad_score", dev)
    if score is None:
        score = torch.empty(B, dtype=torch.float64, device=dev)
    g = {} if grads is None else grads
    for name, shape in (("grad_em", (B, T, C)), ("grad_trans", (C, C)), ("grad_dur", (K, C)),
                        ("grad_p_start", (B, T, C)), ("grad_p_end", (B, T, C))):
        if g.get(name) is not None:
            _need(g[name], torch.float32, name, dev)
            if tuple(g[name].shape) != shape:
                raise TypeError(f"{name} must have shape {shape}")
    if _projections(p_start, p_end, (B, T, C), dev) or g.get("grad_p_start") is not None \
            or g.get("grad_p_end") is not None:
        _check(lib.semicrf_path_score_proj(
            _ptr(em), _ptr(lengths), _ptr(trans), _ptr(dur), _ptr(p_start), _ptr(p_end),
            _ptr(labels), _ptr(seg_start), B, T, C, K, flags, ws.ptr, ws.nbytes, _ptr(grad_score),
            _ptr(score), _ptr(g.get("grad_em")), _ptr(g.get("grad_trans")), _ptr(g.get("grad_dur")),
            _ptr(g.get("grad_p_start")), _ptr(g.get("grad_p_end")), _stream(dev)),
            "semicrf_path_score_proj")
        return score
    _check(lib.semicrf_path_score(_ptr(em), _ptr(lengths), _ptr(trans), _ptr(dur), _ptr(labels),
                                  _ptr(seg_start), B, T, C, K, flags, ws.ptr, ws.nbytes,
                                  _ptr(grad_score), _ptr(score), _ptr(g.get("grad_em")),
                                  _ptr(g.get("grad_trans")), _ptr(g.get("grad_dur")),
                                  _stream(dev)), "semicrf_path_score")
    return score


def get_status(ws: Workspace) -> int:
    """Synchronises the current stream and returns the workspace status word."""
    st = _i(0)
    _check(lib.semicrf_get_status(ws.ptr, _stream(ws.buf.device), ctypes.byref(st)),
           "semicrf_get_status")
    return int(st.value)


def ring_domains(ws: Workspace):
    """Arithmetic of each ring in the last forward on `ws`: a list of 2B ints,
    forward rings then backward rings, 1 = exponential domain, 2 = log
    domain, 0 = not run (synchronises)."""
    B, T, C, K = ws.dims
    out = (ctypes.c_int32 * max(1, 2 * B))()
    _check(lib.semicrf_ring_domains(ws.ptr, ws.nbytes, B, T, C, K, ws.flags,
                                    _stream(ws.buf.device), out), "semicrf_ring_domains")
    return list(out)[:2 * B]


def selftest_bounded_wait(ws: Workspace, spins: int) -> int:
    """Runs the never-completing bounded wait with `spins` polls; returns the
    resulting status word (SEMICRF_ERR_DEVICE_TIMEOUT = 5 expected)."""
    _check(lib.semicrf_selftest_bounded_wait(ws.ptr, ws.nbytes, int(spins), _stream(ws.buf.device)),
           "semicrf_selftest_bounded_wait")
    return get_status(ws)


def selftest_bounds(ws: Workspace) -> int:
    """Bounds-checking build: runs one deliberately out-of-range guarded store
    (skipped by its check) and returns the status word it leaves.  The
    release build raises SemiCRFError(SEMICRF_ERR_UNSUPPORTED)."""
    _check(lib.semicrf_selftest_bounds(ws.ptr, ws.nbytes, _stream(ws.buf.device)),
           "semicrf_selftest_bounds")
    st = _i(0)
    _check(lib.semicrf_get_status(ws.ptr, _stream(ws.buf.device), ctypes.byref(st)),
           "semicrf_get_status")
    return int(st.value)


def profile_enable(on: bool = True):
    """Start (clearing) or stop per-kernel CUDA-event timing inside the library."""
    _check(lib.semicrf_profile_enable(1 if on else 0), "semicrf_profile_enable")


def profile_read(kernel: str):
    """(total device ms, launches) recorded for `kernel` since profile_enable(True)."""
    ms = ctypes.c_double(0.0)
    n = _i(0)
    _check(lib.semicrf_profile_read(kernel.encode(), ctypes.byref(ms), ctypes.byref(n)),
           "semicrf_profile_read")
    return float(ms.value), int(n.value)


def forward_noalloc(em, lengths, trans, dur, center: bool = True, logZ=None,
                    log_domain: bool = False):
    """log Z [B] (float64) through semicrf_forward_noalloc: no workspace, no
    allocation inside the library (the output tensor is allocated here unless
    passed).  Raises SemiCRFError(SEMICRF_ERR_UNSUPPORTED) when the problem
    does not fit the library's fixed scratch array."""
    dev = em.device
    _need(em, torch.float32, "em", dev)
    _need(lengths, torch.int32, "lengths", dev)
    _need(trans, torch.float32, "trans", dev)
    _need(dur, torch.float32, "dur", dev)
    B, T, C = em.shape
    K = dur.shape[0]
    if logZ is None:
        logZ = torch.empty(B, dtype=torch.float64, device=dev)
    _check(lib.semicrf_forward_noalloc(_ptr(em), _ptr(lengths), _ptr(trans), _ptr(dur), B, T, C, K,
                                       _flags(center, True, log_domain), _ptr(logZ),
                                       _stream(dev)),
           "semicrf_forward_noalloc")
    return logZ
