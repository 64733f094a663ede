"""Thin ctypes binding of libcpattn.so (declared in include/cpattn.h).

Argument marshalling only: torch tensors become ``cp_tensor`` descriptors
(device pointer, dtype, sizes, element strides), the current CUDA stream is
passed through, and a non-zero status raises ``CpError``.  Outputs that the
caller does not supply are allocated with torch (memory is torch's job);
every step of the computation runs in the library's CUDA kernels.  There is
no CPU fallback: if the library is not built, the first call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

import torch

# CPATTN_DEBUG=1 selects the bounds-checking build (libcpattn_debug.so,
# compiled with CP_DEBUG): same entry points, every device-side index checked
# against its tensor's extent, failures reported as CP_ERR_BOUNDS by
# cp_last_device_error.
_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                         "libcpattn_debug.so" if os.environ.get("CPATTN_DEBUG") == "1"
                         else "libcpattn.so")

CP_F32, CP_BF16 = 0, 1
MAX_DIMS = 6
MAX_CHUNKS = 512
SEQ_TO_HEAD, HEAD_TO_SEQ = 0, 1

STATUS = {
    0: "CP_OK", -1: "CP_ERR_NULL", -2: "CP_ERR_DTYPE", -3: "CP_ERR_SHAPE", -4: "CP_ERR_ALIGN",
    -5: "CP_ERR_OFFSETS", -6: "CP_ERR_DEGREE", -7: "CP_ERR_CUDA", -8: "CP_ERR_TIMEOUT",
    -9: "CP_ERR_WORKSPACE", -10: "CP_ERR_ALIAS", -11: "CP_ERR_BOUNDS",
}
EXPORTS = ("cp_attn_partial", "cp_attn_partial_merge", "cp_lse_merge", "cp_ring_attention_gathered", "cp_ring_attention", "cp_ulysses_permute",
           "cp_usp_attention", "cp_usp_attention_static", "cp_usp_workspace_bytes",
           "cp_ulysses_anything_permute", "cp_ulysses_anything_attention",
           "cp_ulysses_anything_workspace_bytes", "cp_ring_chunk_offsets",
           "cp_status_string", "cp_last_device_error", "cp_selftest_wait_timeout",
           "cp_selftest_bounds_check")


class CpTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * MAX_DIMS), ("stride", ctypes.c_int64 * MAX_DIMS)]


class CpError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        self.name = STATUS.get(status, str(status))
        super().__init__(f"{where}: {self.name} ({lib().cp_status_string(status).decode()})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (loaded once; raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing: build it with "
                "`python -m context_attention_dits_cp_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.POINTER(CpTensor)
        vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
        L.cp_attn_partial.argtypes = [P, P, P, f32, P, P, vp]
        L.cp_attn_partial_merge.argtypes = [P, P, P, f32, P, P, vp]
        L.cp_lse_merge.argtypes = [P, P, P, P, vp]
        L.cp_ring_attention.argtypes = [P, P, P, ctypes.POINTER(i64), i32, f32, P, P, vp]
        L.cp_ring_attention_gathered.argtypes = [P, P, P, ctypes.POINTER(i64), i32, i32, f32,
                                                 i32, P, P, vp]
        L.cp_ulysses_permute.argtypes = [P, P, i32, i32, vp]
        L.cp_usp_attention.argtypes = [P, P, P, i32, i32, f32, vp, ctypes.c_size_t, P, P, vp]
        L.cp_usp_attention_static.argtypes = [P, P, P, i32, i32, f32, P, P, vp]
        L.cp_usp_workspace_bytes.argtypes = [i64, i64, i64, i64, i32, i32, i32, i32]
        L.cp_usp_workspace_bytes.restype = ctypes.c_size_t
        L.cp_ring_chunk_offsets.argtypes = [i64, i32, ctypes.POINTER(i64)]
        OFF = ctypes.POINTER(i64)
        L.cp_ulysses_anything_permute.argtypes = [P, P, i64, i64, i64, i32, OFF, OFF, i32, vp]
        L.cp_ulysses_anything_attention.argtypes = [P, P, P, i64, i64, i64, i32, OFF, OFF, f32,
                                                    vp, ctypes.c_size_t, P, P, vp]
        L.cp_ulysses_anything_workspace_bytes.argtypes = [i64, i64, i64, i64, i32, i32]
        L.cp_ulysses_anything_workspace_bytes.restype = ctypes.c_size_t
        L.cp_status_string.argtypes = [i32]
        L.cp_status_string.restype = ctypes.c_char_p
        L.cp_last_device_error.argtypes = [vp]
        L.cp_selftest_wait_timeout.argtypes = [i32, vp]
        L.cp_selftest_bounds_check.argtypes = [vp]
        for n in EXPORTS:
            if n not in ("cp_usp_workspace_bytes", "cp_status_string",
                         "cp_ulysses_anything_workspace_bytes"):
                getattr(L, n).restype = ctypes.c_int
        _lib = L
    return _lib


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return CP_F32
    if t.dtype == torch.bfloat16:
        return CP_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def desc(t: Optional[torch.Tensor]) -> Optional[CpTensor]:
    """cp_tensor view of a torch tensor (no copy)."""
    if t is None:
        return None
    if t.dim() > MAX_DIMS:
        raise ValueError("too many dimensions")
    d = CpTensor()
    d.data = t.data_ptr()
    d.dtype = _dtype_code(t)
    d.ndim = t.dim()
    for i in range(t.dim()):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    return d


def _ref(d: Optional[CpTensor]):
    return ctypes.byref(d) if d is not None else None


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(status: int, where: str):
    if status != 0:
        raise CpError(status, where)


def _scale(scale: Optional[float]) -> float:
    return 0.0 if scale is None else float(scale)


# ---------------------------------------------------------------- public calls
def attn_partial(q, k_chunk, v_chunk, scale=None, out=None, lse=None, out_dtype=torch.float32):
    """One ring step: (out, lse) of q against one K/V chunk (cp_attn_partial)."""
    B, S, H, D = q.shape
    out = torch.empty((B, S, H, D), dtype=out_dtype, device=q.device) if out is None else out
    lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device) if lse is None else lse
    dq, dk, dv, do, dl = desc(q), desc(k_chunk), desc(v_chunk), desc(out), desc(lse)
    _check(lib().cp_attn_partial(_ref(dq), _ref(dk), _ref(dv), _scale(scale), _ref(do),
                                 _ref(dl), _stream(q.device)), "cp_attn_partial")
    return out, lse


def attn_partial_merge(q, k_chunk, v_chunk, out_acc, lse_acc, scale=None):
    """One ring step folded into the fp32 accumulator in place
    (cp_attn_partial_merge)."""
    dq, dk, dv, do, dl = desc(q), desc(k_chunk), desc(v_chunk), desc(out_acc), desc(lse_acc)
    _check(lib().cp_attn_partial_merge(_ref(dq), _ref(dk), _ref(dv), _scale(scale), _ref(do),
                                       _ref(dl), _stream(q.device)), "cp_attn_partial_merge")
    return out_acc, lse_acc


def lse_merge(out_acc, lse_acc, out_i, lse_i):
    """In-place fp32 merge of (out_i, lse_i) into (out_acc, lse_acc) (cp_lse_merge)."""
    da, dla, di, dli = desc(out_acc), desc(lse_acc), desc(out_i), desc(lse_i)
    _check(lib().cp_lse_merge(_ref(da), _ref(dla), _ref(di), _ref(dli),
                              _stream(out_acc.device)), "cp_lse_merge")
    return out_acc, lse_acc


def ring_chunk_offsets(S: int, R: int):
    """Ring Anything split of S tokens over R ranks (cp_ring_chunk_offsets)."""
    arr = (ctypes.c_int64 * (R + 1))()
    _check(lib().cp_ring_chunk_offsets(S, R, arr), "cp_ring_chunk_offsets")
    return list(arr)


def ring_attention(q, k, v, chunk_offsets: Sequence[int], scale=None, out=None, lse=None,
                   out_dtype=torch.float32, want_lse=True):
    """The fused ring walk over K/V chunks (cp_ring_attention)."""
    B, S, H, D = q.shape
    out = torch.empty((B, S, H, D), dtype=out_dtype, device=q.device) if out is None else out
    if lse is None and want_lse:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    offs = (ctypes.c_int64 * len(chunk_offsets))(*[int(x) for x in chunk_offsets])
    dq, dk, dv, do, dl = desc(q), desc(k), desc(v), desc(out), desc(lse)
    _check(lib().cp_ring_attention(_ref(dq), _ref(dk), _ref(dv), offs, len(chunk_offsets) - 1,
                                   _scale(scale), _ref(do), _ref(dl), _stream(q.device)),
           "cp_ring_attention")
    return out, lse


def ring_attention_gathered(q, k_gathered, v_gathered, chunk_lengths: Sequence[int],
                            skip_chunk: int = -1, scale=None, out=None, lse=None,
                            accumulate=False, out_dtype=torch.float32, want_lse=True):
    """The ring over the slots [R, B, L, H, D] of a padded K/V all-gather;
    chunk c is rows [0, chunk_lengths[c]) of slot c (cp_ring_attention_gathered).
    With accumulate=True, (out, lse) is an fp32 accumulator updated in place."""
    B, S, H, D = q.shape
    if accumulate and (out is None or lse is None):
        raise ValueError("accumulate=True needs the accumulator (out, lse)")
    out = torch.empty((B, S, H, D), dtype=out_dtype, device=q.device) if out is None else out
    if lse is None and want_lse:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    lens = (ctypes.c_int64 * len(chunk_lengths))(*[int(x) for x in chunk_lengths])
    dq, dk, dv, do, dl = desc(q), desc(k_gathered), desc(v_gathered), desc(out), desc(lse)
    _check(lib().cp_ring_attention_gathered(_ref(dq), _ref(dk), _ref(dv), lens,
                                            len(chunk_lengths), int(skip_chunk), _scale(scale),
                                            1 if accumulate else 0, _ref(do), _ref(dl),
                                            _stream(q.device)),
           "cp_ring_attention_gathered")
    return out, lse


def ulysses_permute(x, degree: int, direction: int, y=None):
    """Ulysses all-to-all as a layout permutation (cp_ulysses_permute)."""
    U, B, S1, H1, D = x.shape
    if y is None:
        shape = (U, B, S1 * U, H1 // U, D) if direction == SEQ_TO_HEAD else (U, B, S1 // U, H1 * U, D)
        y = torch.empty(shape, dtype=x.dtype, device=x.device)
    dx, dy = desc(x), desc(y)
    _check(lib().cp_ulysses_permute(_ref(dx), _ref(dy), int(degree), int(direction),
                                    _stream(x.device)), "cp_ulysses_permute")
    return y


def usp_workspace_bytes(B, S, H, D, in_dtype, out_dtype, ring_degree, ulysses_degree) -> int:
    code = lambda dt: CP_F32 if dt == torch.float32 else CP_BF16
    return int(lib().cp_usp_workspace_bytes(B, S, H, D, code(in_dtype), code(out_dtype),
                                            ring_degree, ulysses_degree))


def usp_attention(q_shards, k_shards, v_shards, ring_degree: int, ulysses_degree: int,
                  scale=None, out=None, lse=None, workspace=None, out_dtype=torch.float32,
                  want_lse=True):
    """Unified (Ulysses x Ring) attention on shard-major inputs (cp_usp_attention)."""
    G, B, Sg, H, D = q_shards.shape
    S = G * Sg
    out = torch.empty_like(q_shards, dtype=out_dtype) if out is None else out
    if lse is None and want_lse:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q_shards.device)
    need = usp_workspace_bytes(B, S, H, D, q_shards.dtype, out.dtype, ring_degree, ulysses_degree)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q_shards.device)
    dq, dk, dv, do, dl = desc(q_shards), desc(k_shards), desc(v_shards), desc(out), desc(lse)
    _check(lib().cp_usp_attention(_ref(dq), _ref(dk), _ref(dv), int(ring_degree),
                                  int(ulysses_degree), _scale(scale),
                                  ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
                                  _ref(do), _ref(dl), _stream(q_shards.device)),
           "cp_usp_attention")
    return out, lse


def _offsets(offs):
    return (ctypes.c_int64 * len(offs))(*[int(x) for x in offs])


def ulysses_anything_permute(x, B, H, D, seq_offsets, head_offsets, direction, y=None):
    """Uneven Ulysses all-to-all on flat rank buffers (cp_ulysses_anything_permute)."""
    y = torch.empty_like(x) if y is None else y
    U = len(seq_offsets) - 1
    _check(lib().cp_ulysses_anything_permute(_ref(desc(x)), _ref(desc(y)), int(B), int(H), int(D),
                                             U, _offsets(seq_offsets), _offsets(head_offsets),
                                             int(direction), _stream(x.device)),
           "cp_ulysses_anything_permute")
    return y


def ulysses_anything_attention(q, k, v, B, H, D, seq_offsets, head_offsets, scale=None,
                               out=None, lse=None, workspace=None, out_dtype=torch.float32,
                               want_lse=True):
    """Ulysses Anything attention on flat sequence-side buffers
    (cp_ulysses_anything_attention)."""
    S = int(seq_offsets[-1])
    U = len(seq_offsets) - 1
    out = torch.empty(q.shape, dtype=out_dtype, device=q.device) if out is None else out
    if lse is None and want_lse:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    if workspace is None:
        code = lambda dt: CP_F32 if dt == torch.float32 else CP_BF16
        need = int(lib().cp_ulysses_anything_workspace_bytes(B, S, H, D, code(q.dtype),
                                                             code(out.dtype)))
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _check(lib().cp_ulysses_anything_attention(
        _ref(desc(q)), _ref(desc(k)), _ref(desc(v)), int(B), int(H), int(D), U,
        _offsets(seq_offsets), _offsets(head_offsets), _scale(scale),
        ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), _ref(desc(out)),
        _ref(desc(lse)), _stream(q.device)), "cp_ulysses_anything_attention")
    return out, lse


USP_STATIC_SCRATCH_BYTES = 64 * 1024 * 1024


def usp_attention_static(q_shards, k_shards, v_shards, ring_degree: int, ulysses_degree: int,
                         scale=None, out=None, lse=None, out_dtype=torch.float32, want_lse=True):
    """usp_attention without a workspace argument, for callers that cannot
    allocate device memory (cp_usp_attention_static): the library's fixed
    64 MiB device array serves as the workspace; larger problems are
    rejected with CP_ERR_WORKSPACE.  Pass preallocated `out`/`lse` to make
    the call allocate nothing at all."""
    G, B, Sg, H, D = q_shards.shape
    S = G * Sg
    out = torch.empty_like(q_shards, dtype=out_dtype) if out is None else out
    if lse is None and want_lse:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q_shards.device)
    dq, dk, dv, do, dl = desc(q_shards), desc(k_shards), desc(v_shards), desc(out), desc(lse)
    _check(lib().cp_usp_attention_static(_ref(dq), _ref(dk), _ref(dv), int(ring_degree),
                                         int(ulysses_degree), _scale(scale), _ref(do), _ref(dl),
                                         _stream(q_shards.device)),
           "cp_usp_attention_static")
    return out, lse


def last_device_error(device=None) -> int:
    """Synchronises the current stream; CP_ERR_TIMEOUT if a bounded wait gave
    up, CP_ERR_BOUNDS if a debug-build bounds check failed."""
    dev = torch.device("cuda") if device is None else device
    return int(lib().cp_last_device_error(_stream(dev)))


def selftest_wait_timeout(spin_limit: int = 4096, device=None) -> int:
    dev = torch.device("cuda") if device is None else device
    st = int(lib().cp_selftest_wait_timeout(int(spin_limit), _stream(dev)))
    _check(st, "cp_selftest_wait_timeout")
    return last_device_error(dev)


def selftest_bounds_check(device=None) -> int:
    """One deliberately failing device-side bounds check; returns what
    cp_last_device_error reports afterwards (CP_ERR_BOUNDS on the debug
    build, CP_OK on the release build)."""
    dev = torch.device("cuda") if device is None else device
    _check(int(lib().cp_selftest_bounds_check(_stream(dev))), "cp_selftest_bounds_check")
    return last_device_error(dev)


def is_debug_build() -> bool:
    """True when the bounds-checking library (CPATTN_DEBUG=1) is loaded."""
    return os.path.basename(_LIB_PATH) == "libcpattn_debug.so"


def attention_flops(B, H, S_q, S_kv, D) -> float:
    """4*B*H*S_q*S_kv*D: QK^T and PV, two flops per multiply-add."""
    return 4.0 * B * H * S_q * S_kv * D


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
