"""Thin ctypes binding over libgdn.so (C ABI in include/gdn.h).

Argument marshalling only: every step of the mixer runs in the library's CUDA kernels.
Tensors are PyTorch CUDA tensors used as device memory; the stream is the current torch
stream unless one is given. There is no fallback: if libgdn.so is missing or a call fails,
an exception is raised.

Passages the entry points follow: the Gated DeltaNet mixer and its recurrent-state
commit / rollback ("Lithos-metal: Qwen3.8-27B on 40-core M5 Max", table "GDN mixer" and
the runtime paragraph) over a verify block of 7 drafts + 1 anchor ("Qwen 3.8 27B mac m5:
200 tok/s, audited", DSpark section).
"""
import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libgdn.so")

GDN_F32, GDN_BF16 = 0, 1
STATUS_BAD_ACCEPT = 1
GDN_LAUNCH_PDL = 1   # gdn_shape.launch_flags: programmatic dependent launch (include/gdn.h)


class GdnError(RuntimeError):
    """A libgdn call returned a non-zero gdn_status."""

    def __init__(self, status: int, message: str):
        super().__init__("gdn status %d: %s" % (status, message))
        self.status = status


class _Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("T", ctypes.c_int32), ("H_k", ctypes.c_int32),
                ("H_v", ctypes.c_int32), ("d_k", ctypes.c_int32), ("d_v", ctypes.c_int32),
                ("in_dtype", ctypes.c_int32), ("out_dtype", ctypes.c_int32),
                ("l2_eps", ctypes.c_float), ("scale", ctypes.c_float),
                ("status_word", ctypes.c_void_p), ("launch_flags", ctypes.c_uint32)]


class _AcceptShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("T", ctypes.c_int32), ("V", ctypes.c_int32),
                ("logits_dtype", ctypes.c_int32), ("sampled", ctypes.c_int32),
                ("temperature", ctypes.c_float)]


_lib = None
_VP = ctypes.c_void_p


def library_path() -> str:
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError("libgdn.so not built at %s: run `python -m gated_deltanet_mixer_verify_b200"
                          ".build` (or __graft_entry__.build())" % _LIB_PATH)
    lib = ctypes.CDLL(_LIB_PATH)
    S = ctypes.POINTER(_Shape)
    lib.gdn_verify_step.argtypes = [S] + [_VP] * 13
    lib.gdn_commit.argtypes = [S] + [_VP] * 5
    lib.gdn_decode_step.argtypes = [S] + [_VP] * 10
    lib.gdn_commit_and_verify.argtypes = [S, ctypes.c_int32] + [_VP] * 14
    lib.gdn_chunk_prefill.argtypes = ([S, ctypes.c_int32] + [_VP] * 11 + [ctypes.c_size_t, _VP])
    lib.gdn_chunk_prefill_noalloc.argtypes = [S, ctypes.c_int32] + [_VP] * 11
    lib.gdn_chunk_prefill_prepare.argtypes = [S, ctypes.c_int32] + [_VP] * 7 + [ctypes.c_size_t, _VP]
    lib.gdn_chunk_prefill_scan.argtypes = [S, ctypes.c_int32] + [_VP] * 5 + [ctypes.c_size_t, _VP]
    lib.gdn_short_conv.argtypes = [S, ctypes.c_int32] + [_VP] * 11
    lib.gdn_selftest_bounded_wait.argtypes = [_VP, ctypes.c_uint32, _VP]
    lib.gdn_selftest_accept_wait.argtypes = [_VP, _VP, ctypes.c_uint32, _VP]
    A = ctypes.POINTER(_AcceptShape)
    lib.gdn_accept.argtypes = [A] + [_VP] * 7 + [ctypes.c_size_t, _VP]
    lib.gdn_accept_workspace_bytes.argtypes = [A]
    lib.gdn_accept_workspace_bytes.restype = ctypes.c_size_t
    lib.gdn_verify_step_gated.argtypes = [S] + [_VP] * 12 + [ctypes.c_float] + [_VP] * 3
    lib.gdn_gated_rmsnorm.argtypes = [ctypes.c_int64, ctypes.c_int32, _VP, ctypes.c_int32, _VP, ctypes.c_int32,
                                      _VP, ctypes.c_float, _VP, ctypes.c_int32, _VP]
    for fn in ("gdn_verify_step", "gdn_commit", "gdn_decode_step", "gdn_commit_and_verify", "gdn_chunk_prefill",
               "gdn_chunk_prefill_noalloc", "gdn_chunk_prefill_prepare", "gdn_chunk_prefill_scan",
               "gdn_short_conv", "gdn_verify_step_gated", "gdn_gated_rmsnorm", "gdn_accept",
               "gdn_selftest_bounded_wait", "gdn_selftest_accept_wait"):
        getattr(lib, fn).restype = ctypes.c_int
    lib.gdn_stash_bytes.argtypes = [S]
    lib.gdn_stash_bytes.restype = ctypes.c_size_t
    lib.gdn_chunk_prefill_workspace_bytes.argtypes = [S, ctypes.c_int32]
    lib.gdn_chunk_prefill_workspace_bytes.restype = ctypes.c_size_t
    lib.gdn_chunk_prefill_pieces.argtypes = [ctypes.c_int64, ctypes.c_int32]
    lib.gdn_chunk_prefill_pieces.restype = ctypes.c_int32
    lib.gdn_status_string.argtypes = [ctypes.c_int]
    lib.gdn_status_string.restype = ctypes.c_char_p
    lib.gdn_last_error.argtypes = []
    lib.gdn_last_error.restype = ctypes.c_char_p
    lib.gdn_abi_version.argtypes = []
    lib.gdn_abi_version.restype = ctypes.c_int32
    lib.gdn_last_verify_kernel.argtypes = []
    lib.gdn_last_verify_kernel.restype = ctypes.c_char_p
    _lib = lib
    return lib


def lib():
    """The loaded ctypes library (raises ImportError if it was never built)."""
    return _load()


def last_verify_kernel() -> str:
    """Name of the kernel this thread's last verify / decode call launched (gdn_last_verify_kernel)."""
    return _load().gdn_last_verify_kernel().decode()


def _check(rc: int):
    if rc != 0:
        raise GdnError(rc, _load().gdn_last_error().decode())


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return GDN_F32
    if dt == torch.bfloat16:
        return GDN_BF16
    raise TypeError("unsupported dtype %s (float32 or bfloat16)" % dt)


def make_shape(B, T, H_k, H_v, d_k, d_v, in_dtype=torch.bfloat16, out_dtype=torch.float32,
               l2_eps=1e-6, scale=1.0, status_word: Optional[torch.Tensor] = None, launch_flags=0) -> _Shape:
    sw = status_word.data_ptr() if status_word is not None else None
    return _Shape(B, T, H_k, H_v, d_k, d_v, _dtype_code(in_dtype), _dtype_code(out_dtype),
                  float(l2_eps), float(scale), sw, int(launch_flags))


def _ptrs(*ts):
    """Device pointers of the given tensors (None stays None), after the checks the C ABI cannot
    make on a bare pointer: a CUDA tensor, contiguous, on the current device (kernels launch on
    the current device's stream, so a tensor on another GPU would be read and written through a
    peer address by the wrong device). The current device is asked for once per call."""
    cur = None
    out = []
    for t in ts:
        if t is None:
            out.append(None)
            continue
        if not t.is_cuda:
            raise ValueError("expected a CUDA tensor")
        if not t.is_contiguous():
            raise ValueError("expected a contiguous tensor")
        if cur is None:
            cur = torch.cuda.current_device()
        d = t.get_device()
        if d != cur:
            raise ValueError("tensor is on cuda:%d but the current CUDA device is cuda:%d; call under "
                             "torch.cuda.device(%d)" % (d, cur, d))
        out.append(t.data_ptr())
    return out


def _ptr(t: Optional[torch.Tensor]):
    return _ptrs(t)[0]


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _shape_from(q, k, v, status_word, l2_eps, scale, out_dtype, launch_flags=0) -> _Shape:
    B, T, H_k, d_k = k.shape
    H_v, d_v = v.shape[2], v.shape[3]
    if q.shape != k.shape or v.shape[:2] != (B, T):
        raise ValueError("q, k [B,T,H_k,d_k] and v [B,T,H_v,d_v] disagree")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share a dtype")
    return make_shape(B, T, H_k, H_v, d_k, d_v, q.dtype, out_dtype, l2_eps, scale, status_word, launch_flags)


def _types(f32=(), i32=()):
    """fp32 (states, stashes, gate parameters, weights) and int32 (counts) arguments, as
    (name, tensor-or-None) pairs."""
    for name, t in f32:
        if t is not None and t.dtype != torch.float32:
            raise TypeError("%s must be float32, not %s" % (name, t.dtype))
    for name, t in i32:
        if t is not None and t.dtype != torch.int32:
            raise TypeError("%s must be int32, not %s" % (name, t.dtype))


def _dtypes(q, a, b, A_log, dt_bias, o=None, out_dtype=None, f32=(), i32=()):
    """Element types the C ABI takes: a, b in q's dtype; A_log, dt_bias and the f32 pairs fp32;
    the i32 pairs int32; o (when given) in out_dtype."""
    if a.dtype != q.dtype or b.dtype != q.dtype:
        raise TypeError("a and b must have q's dtype (%s)" % q.dtype)
    _types((("A_log", A_log), ("dt_bias", dt_bias)) + tuple(f32), i32)
    if o is not None and out_dtype is not None and o.dtype != out_dtype:
        raise TypeError("o is %s but out_dtype is %s" % (o.dtype, out_dtype))


def stash_bytes(B, T, H_k, H_v, d_k, d_v) -> int:
    """Bytes of stash a two-phase verify writes for this shape."""
    return int(_load().gdn_stash_bytes(ctypes.byref(make_shape(B, T, H_k, H_v, d_k, d_v))))


def prefill_workspace_bytes(B, T, H_k, H_v, d_k, d_v, chunk=64) -> int:
    """Bytes of workspace gdn_chunk_prefill needs for this shape."""
    return int(_load().gdn_chunk_prefill_workspace_bytes(
        ctypes.byref(make_shape(B, T, H_k, H_v, d_k, d_v)), chunk))


def chunk_prefill_pieces(T, chunk=64) -> int:
    """Pieces chunk_prefill splits a T-token prompt into (one preparation and one scan launch
    each); -1 for an unsupported chunk."""
    return int(_load().gdn_chunk_prefill_pieces(T, chunk))


def verify_step(q, k, v, a, b, A_log, dt_bias, state_in, state_out=None, accept_len=None, o=None,
                stash=None, l2_eps=1e-6, scale=1.0, status_word=None, out_dtype=torch.float32,
                stream=None, pdl=False):
    """One verify block: o for all T tokens; with ``accept_len`` the committed state S_L goes
    to ``state_out`` (default: in place into ``state_in``); without it, ``stash`` (a float32
    CUDA tensor of stash_bytes()/4 elements) receives what :func:`commit` needs. ``pdl``:
    programmatic dependent launch (GDN_LAUNCH_PDL in include/gdn.h). Returns o."""
    sh = _shape_from(q, k, v, status_word, l2_eps, scale, out_dtype, GDN_LAUNCH_PDL if pdl else 0)
    _dtypes(q, a, b, A_log, dt_bias, o, out_dtype,
            f32=(("state_in", state_in), ("state_out", state_out), ("stash", stash)), i32=(("accept_len", accept_len),))
    if o is None:
        o = torch.empty(v.shape, dtype=out_dtype, device=v.device)
    if accept_len is not None and state_out is None:
        state_out = state_in
    _check(_load().gdn_verify_step(ctypes.byref(sh), *_ptrs(q, k, v, a, b, A_log, dt_bias, state_in, state_out,
                                                           accept_len, o, stash), _stream(stream)))
    return o


def commit(state_in, stash, accept_len, T, H_k, d_k=None, state_out=None, status_word=None,
           stream=None):
    """Second phase of a two-phase verify: state_out = S_L from state_in and the stash.
    ``T`` and ``H_k`` are the verify call's; state_out defaults to state_in (in place)."""
    B, H_v, d_v, dk = state_in.shape
    sh = make_shape(B, T, H_k, H_v, dk if d_k is None else d_k, d_v, status_word=status_word)
    _types(f32=(("state_in", state_in), ("state_out", state_out), ("stash", stash)), i32=(("accept_len", accept_len),))
    if state_out is None:
        state_out = state_in
    _check(_load().gdn_commit(ctypes.byref(sh), *_ptrs(state_in, state_out, stash, accept_len), _stream(stream)))
    return state_out


def commit_and_verify(q, k, v, a, b, A_log, dt_bias, state, prev_stash, prev_accept_len, prev_T,
                      accept_len=None, o=None, stash=None, l2_eps=1e-6, scale=1.0, status_word=None,
                      out_dtype=torch.float32, stream=None):
    """Commit-on-next-verify: ``state`` holds the state the previous (two-phase) block started
    from; its stash and device accept counts are applied on the way in. With ``accept_len``
    the state ends committed at this block's counts; without it the state ends at the
    committed previous block and ``stash`` receives this block's. Returns o."""
    sh = _shape_from(q, k, v, status_word, l2_eps, scale, out_dtype)
    _dtypes(q, a, b, A_log, dt_bias, o, out_dtype, f32=(("state", state), ("prev_stash", prev_stash), ("stash", stash)),
            i32=(("prev_accept_len", prev_accept_len), ("accept_len", accept_len)))
    if o is None:
        o = torch.empty(v.shape, dtype=out_dtype, device=v.device)
    _check(_load().gdn_commit_and_verify(ctypes.byref(sh), int(prev_T),
                                         *_ptrs(q, k, v, a, b, A_log, dt_bias, state, prev_stash,
                                                prev_accept_len, accept_len, o, stash),
                                         _stream(stream)))
    return o


def verify_step_gated(q, k, v, a, b, A_log, dt_bias, state_in, state_out, accept_len, norm_z, norm_w,
                      norm_eps=1e-6, o=None, stash=None, l2_eps=1e-6, scale=1.0, status_word=None,
                      out_dtype=torch.float32, stream=None):
    """verify_step whose outputs are o / sqrt(mean(o^2) + norm_eps) * norm_w * silu(norm_z) per
    (token, value head); norm_z has v's shape and dtype, norm_w is [d_v] fp32. Returns o."""
    sh = _shape_from(q, k, v, status_word, l2_eps, scale, out_dtype)
    _dtypes(q, a, b, A_log, dt_bias, o, out_dtype,
            f32=(("state_in", state_in), ("state_out", state_out), ("stash", stash), ("norm_w", norm_w)),
            i32=(("accept_len", accept_len),))
    if norm_z.shape != v.shape or norm_z.dtype != v.dtype:
        raise ValueError("norm_z must have v's shape and dtype")
    if o is None:
        o = torch.empty(v.shape, dtype=out_dtype, device=v.device)
    ptrs = _ptrs(q, k, v, a, b, A_log, dt_bias, state_in, state_out, accept_len, norm_z, norm_w, o, stash)
    _check(_load().gdn_verify_step_gated(ctypes.byref(sh), *ptrs[:12], float(norm_eps), *ptrs[12:], _stream(stream)))
    return o


def gated_rmsnorm(x, z, w, eps=1e-6, y=None, out_dtype=None, stream=None):
    """y = x / sqrt(mean(x^2) + eps) * w * silu(z) over the last axis (x, z [..., d]; w [d] fp32).
    y may be x (in place). Returns y."""
    d = x.shape[-1]
    if z.shape != x.shape or w.shape != (d,):
        raise ValueError("x, z [..., d] and w [d] disagree")
    if y is None:
        y = torch.empty(x.shape, dtype=out_dtype or x.dtype, device=x.device)
    _check(_load().gdn_gated_rmsnorm(x.numel() // d if d else 0, d, _ptr(x), _dtype_code(x.dtype), _ptr(z),
                                     _dtype_code(z.dtype), _ptr(w), float(eps), _ptr(y), _dtype_code(y.dtype),
                                     _stream(stream)))
    return y


def _accept_shape(B, T, V, dtype, sampled, temperature) -> _AcceptShape:
    return _AcceptShape(B, T, V, _dtype_code(dtype), int(bool(sampled)), float(temperature))


def accept_workspace_bytes(B, T, V, sampled, dtype=torch.bfloat16) -> int:
    """Bytes of workspace :func:`accept` needs."""
    sh = _accept_shape(B, T, V, dtype, sampled, 1.0)
    return int(_load().gdn_accept_workspace_bytes(ctypes.byref(sh)))


def accept(target, tokens, draft=None, uniforms=None, temperature=1.0, workspace=None, accept_len=None,
           next_token=None, stream=None):
    """Device-side acceptance of verify blocks. target [B, T, V] logits (bf16 or fp32), tokens
    [B, T] int32 (the anchor, then the drafts); sampled mode when draft [B, T-1, V] and uniforms
    [B, T] fp32 are given, greedy otherwise. Returns (accept_len [B], next_token [B]) int32."""
    B, T, V = target.shape
    sampled = uniforms is not None
    sh = _accept_shape(B, T, V, target.dtype, sampled, temperature)
    if workspace is None:
        workspace = torch.empty(max(accept_workspace_bytes(B, T, V, sampled, target.dtype), 16),
                                dtype=torch.uint8, device=target.device)
    if accept_len is None:
        accept_len = torch.empty(B, dtype=torch.int32, device=target.device)
    if next_token is None:
        next_token = torch.empty(B, dtype=torch.int32, device=target.device)
    _check(_load().gdn_accept(ctypes.byref(sh),
                              *_ptrs(target, draft, tokens, uniforms, accept_len, next_token, workspace),
                              workspace.numel() * workspace.element_size(), _stream(stream)))
    return accept_len, next_token


def selftest_bounded_wait(status_word, polls=1024, stream=None):
    """Run the library's bounded-wait failure path once: a wait that nothing completes gives up
    after `polls` polls and ORs the wait-timeout bit (2) into status_word (device int32)."""
    _check(_load().gdn_selftest_bounded_wait(_ptr(status_word), int(polls), _stream(stream)))


def selftest_accept_wait(status_word, next_token, polls=1024, stream=None):
    """Run the acceptance draw kernel's flag wait once with a flag nothing raises: it gives up
    after `polls` polls, ORs the wait-timeout bit (2) into status_word and writes 0 to
    next_token[0] (both device int32)."""
    _check(_load().gdn_selftest_accept_wait(*_ptrs(status_word, next_token), int(polls), _stream(stream)))


def conv_channels(H_k, H_v, d_k, d_v) -> int:
    """Channels of the short convolution: q | k | v."""
    return 2 * H_k * d_k + H_v * d_v


def short_conv(q, k, v, conv_w, hist_in, hist_out=None, accept_len=None, outputs=True,
               q_out=None, k_out=None, v_out=None, status_word=None, stream=None):
    """Causal short convolution of q, k, v (channels q | k | v, conv_w [C, K] fp32, SiLU) with
    the history hist_in [B, K-1, C] (dtype of q), rewound into hist_out at accept_len (device
    int32 [B]; None: all T accepted). hist_out may be hist_in (in place) or None (not written).
    outputs=False only rewinds the history. Returns (q', k', v') or None."""
    sh = _shape_from(q, k, v, status_word, 1e-6, 1.0, torch.float32)
    if hist_in.dtype != q.dtype or (hist_out is not None and hist_out.dtype != q.dtype):
        raise TypeError("the history has the dtype of q, k, v")
    if outputs:
        q_out = torch.empty_like(q) if q_out is None else q_out
        k_out = torch.empty_like(k) if k_out is None else k_out
        v_out = torch.empty_like(v) if v_out is None else v_out
    else:
        q_out = k_out = v_out = None
    _check(_load().gdn_short_conv(ctypes.byref(sh), int(conv_w.shape[1]) if conv_w is not None else
                                  int(hist_in.shape[1]) + 1,
                                  *_ptrs(q, k, v, conv_w, hist_in, hist_out, accept_len, q_out, k_out, v_out),
                                  _stream(stream)))
    return (q_out, k_out, v_out) if outputs else None


def decode_step(q, k, v, a, b, A_log, dt_bias, state, o=None, l2_eps=1e-6, scale=1.0,
                status_word=None, out_dtype=torch.float32, stream=None, pdl=False):
    """One plain decoding token (T = 1): returns o and updates ``state`` in place. ``pdl``:
    programmatic dependent launch (GDN_LAUNCH_PDL in include/gdn.h)."""
    sh = _shape_from(q, k, v, status_word, l2_eps, scale, out_dtype, GDN_LAUNCH_PDL if pdl else 0)
    _dtypes(q, a, b, A_log, dt_bias, o, out_dtype, f32=(("state", state),))
    if o is None:
        o = torch.empty(v.shape, dtype=out_dtype, device=v.device)
    _check(_load().gdn_decode_step(ctypes.byref(sh), *_ptrs(q, k, v, a, b, A_log, dt_bias, state, o),
                                   _stream(stream)))
    return o


def chunk_prefill(q, k, v, a, b, A_log, dt_bias, state_in=None, state_out=None, o=None, chunk=64,
                  workspace=None, l2_eps=1e-6, scale=1.0, status_word=None,
                  out_dtype=torch.float32, stream=None):
    """The mixer over a whole prompt: returns (o, state_out). ``state_in`` None = zero state.
    ``workspace`` (uint8 CUDA tensor) must hold prefill_workspace_bytes(); it is allocated
    here when not given. A prompt of 64 chunks or more runs in chunk_prefill_pieces(T) pieces,
    the scans on a stream of the library's own, joined back to ``stream`` before it returns."""
    sh = _shape_from(q, k, v, status_word, l2_eps, scale, out_dtype)
    _dtypes(q, a, b, A_log, dt_bias, o, out_dtype, f32=(("state_in", state_in), ("state_out", state_out)))
    B, T, H_k, d_k = k.shape
    H_v, d_v = v.shape[2], v.shape[3]
    if o is None:
        o = torch.empty(v.shape, dtype=out_dtype, device=v.device)
    if state_out is None:
        state_out = torch.empty((B, H_v, d_v, d_k), dtype=torch.float32, device=v.device)
    need = int(_load().gdn_chunk_prefill_workspace_bytes(ctypes.byref(sh), chunk))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=v.device)
    wbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(_load().gdn_chunk_prefill(ctypes.byref(sh), chunk,
                                     *_ptrs(q, k, v, a, b, A_log, dt_bias, state_in, state_out, o, workspace), wbytes,
                                     _stream(stream)))
    return o, state_out


def _nbytes(t: Optional[torch.Tensor]) -> int:
    return t.numel() * t.element_size() if t is not None else 0


def chunk_prefill_prepare(q, k, a, b, A_log, dt_bias, workspace, H_v=None, d_v=None, chunk=64,
                          l2_eps=1e-6, scale=1.0, status_word=None, out_dtype=torch.float32,
                          stream=None):
    """First phase of chunk_prefill, over the whole prompt: the state-independent per-chunk
    operators of the prompt into ``workspace`` (uint8 CUDA tensor of
    prefill_workspace_bytes()). H_v defaults to a.shape[2], d_v to d_k."""
    B, T, H_k, d_k = k.shape
    H_v = a.shape[2] if H_v is None else H_v
    d_v = d_k if d_v is None else d_v
    sh = make_shape(B, T, H_k, H_v, d_k, d_v, q.dtype, out_dtype, l2_eps, scale, status_word)
    _dtypes(q, a, b, A_log, dt_bias)
    _check(_load().gdn_chunk_prefill_prepare(ctypes.byref(sh), chunk, *_ptrs(q, k, a, b, A_log, dt_bias, workspace),
                                             _nbytes(workspace), _stream(stream)))


def chunk_prefill_scan(v, workspace, H_k, state_in=None, state_out=None, o=None, d_k=None, chunk=64,
                       status_word=None, out_dtype=torch.float32, stream=None):
    """Second phase of chunk_prefill, over the whole prompt: the scan over the chunks of a
    prepared ``workspace``. Returns (o, state_out); ``H_k`` (and d_k, default d_v) must match
    the prepare call."""
    B, T, H_v, d_v = v.shape
    d_k = d_v if d_k is None else d_k
    sh = make_shape(B, T, H_k, H_v, d_k, d_v, v.dtype, out_dtype, status_word=status_word)
    _types(f32=(("state_in", state_in), ("state_out", state_out)))
    if o is not None and o.dtype != out_dtype:
        raise TypeError("o is %s but out_dtype is %s" % (o.dtype, out_dtype))
    if o is None:
        o = torch.empty(v.shape, dtype=out_dtype, device=v.device)
    if state_out is None:
        state_out = torch.empty((B, H_v, d_v, d_k), dtype=torch.float32, device=v.device)
    _check(_load().gdn_chunk_prefill_scan(ctypes.byref(sh), chunk, *_ptrs(v, state_in, state_out, o, workspace),
                                          _nbytes(workspace), _stream(stream)))
    return o, state_out


NOALLOC_SCRATCH_BYTES = 64 << 20


def chunk_prefill_noalloc(q, k, v, a, b, A_log, dt_bias, state_in=None, state_out=None, o=None,
                          chunk=64, l2_eps=1e-6, scale=1.0, status_word=None,
                          out_dtype=torch.float32, stream=None):
    """chunk_prefill without a workspace, for callers that cannot allocate device memory.

    The library's fixed device scratch (NOALLOC_SCRATCH_BYTES per GPU) is used instead; shapes
    that need more raise GdnError. Calls that overlap on the GPU share that scratch and race.
    ``o`` and ``state_out`` are the caller's; they are only created here when omitted."""
    sh = _shape_from(q, k, v, status_word, l2_eps, scale, out_dtype)
    _dtypes(q, a, b, A_log, dt_bias, o, out_dtype, f32=(("state_in", state_in), ("state_out", state_out)))
    B, T, H_k, d_k = k.shape
    H_v, d_v = v.shape[2], v.shape[3]
    if o is None:
        o = torch.empty(v.shape, dtype=out_dtype, device=v.device)
    if state_out is None:
        state_out = torch.empty((B, H_v, d_v, d_k), dtype=torch.float32, device=v.device)
    _check(_load().gdn_chunk_prefill_noalloc(ctypes.byref(sh), chunk,
                                             *_ptrs(q, k, v, a, b, A_log, dt_bias, state_in, state_out, o),
                                             _stream(stream)))
    return o, state_out
