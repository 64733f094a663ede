"""The C-ABI library on the host: it loads, exports every declared symbol, and
rejects bad arguments with the documented status codes before touching the
GPU (no device is needed for any of these)."""
import ctypes
import os
import re

import pytest

from context_attention_dits_cp_b200 import binding as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x100000   # never dereferenced: validation fails before any launch


def _declared():
    src = open(os.path.join(ROOT, "include", "cpattn.h")).read()
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(cp_\w+)\(", src, re.M)))


def test_header_declares_every_binding_export():
    assert _declared() == sorted(bd.EXPORTS)


def test_library_loads_and_exports_all_symbols():
    L = bd.lib()
    for name in _declared():
        assert hasattr(L, name), name


def test_debug_library_exports_the_same_symbols():
    """libcpattn_debug.so (CP_DEBUG: device-side bounds checks) is the same
    C-ABI: every declared entry point is there."""
    path = os.path.join(os.path.dirname(bd.__file__), "libcpattn_debug.so")
    assert os.path.exists(path), "build() makes the debug library too"
    D = ctypes.CDLL(path)
    for name in _declared():
        assert hasattr(D, name), name


def _t(shape, dtype=bd.CP_BF16, data=FAKE, strides=None):
    d = bd.CpTensor()
    d.data = data
    d.dtype = dtype
    d.ndim = len(shape)
    if strides is None:
        strides, acc = [], 1
        for s in reversed(shape):
            strides.insert(0, acc)
            acc *= s
    for i, (s, st) in enumerate(zip(shape, strides)):
        d.shape[i] = s
        d.stride[i] = st
    return d


def _partial(q, k, v, out, lse):
    r = lambda x: ctypes.byref(x) if x is not None else None
    return bd.lib().cp_attn_partial(r(q), r(k), r(v), 0.0, r(out), r(lse), None)


def _ok_args(D=128, dtype=bd.CP_BF16):
    q = _t([1, 256, 2, D], dtype, FAKE)
    k = _t([1, 300, 2, D], dtype, FAKE + (1 << 24))
    v = _t([1, 300, 2, D], dtype, FAKE + (2 << 24))
    out = _t([1, 256, 2, D], bd.CP_F32, FAKE + (3 << 24))
    lse = _t([1, 2, 256], bd.CP_F32, FAKE + (4 << 24))
    return q, k, v, out, lse


def test_status_strings():
    for code, name in bd.STATUS.items():
        s = bd.lib().cp_status_string(code).decode()
        assert s and s != "unknown status", name
    assert bd.lib().cp_status_string(12345).decode() == "unknown status"


def test_attn_partial_argument_errors():
    q, k, v, out, lse = _ok_args()
    assert _partial(None, k, v, out, lse) == -1                   # NULL
    assert _partial(q, k, v, out, None) == -1                     # lse required
    bad = _t([1, 256, 2, 96]); assert _partial(bad, k, v, out, lse) == -3   # D
    assert _partial(q, _t([1, 300, 3, 128]), v, out, lse) == -3   # H mismatch
    assert _partial(q, k, _t([1, 299, 2, 128]), out, lse) == -3   # S_kv mismatch
    assert _partial(q, k, v, out, _t([1, 2, 255], bd.CP_F32)) == -3
    assert _partial(q, _t([1, 300, 2, 128], bd.CP_F32), v, out, lse) == -2  # mixed dtype
    assert _partial(q, k, v, out, _t([1, 2, 256], bd.CP_BF16)) == -2       # lse dtype
    mis = _t([1, 256, 2, 128], bd.CP_BF16, FAKE + 2)
    assert _partial(mis, k, v, out, lse) == -4                    # TMA base alignment
    odd = _t([1, 256, 2, 128], bd.CP_BF16, FAKE, strides=[256 * 2 * 130, 2 * 130, 130, 1])
    assert _partial(odd, k, v, out, lse) == -4                    # TMA stride alignment
    nc = _t([1, 256, 2, 128], bd.CP_BF16, FAKE, strides=[65536, 256, 128, 2])
    assert _partial(nc, k, v, out, lse) == -4                     # D not contiguous
    alias = _t([1, 256, 2, 128], bd.CP_F32, FAKE)                 # out on top of q
    assert _partial(q, k, v, alias, lse) == -10


def test_self_overlapping_outputs_are_rejected():
    """An output that maps two elements to one address (a broadcast dim, or
    dims that interleave) is refused before any launch."""
    q, k, v, out, lse = _ok_args()
    L = bd.lib()
    r = ctypes.byref
    bcast = _t([1, 256, 2, 128], bd.CP_F32, FAKE + (3 << 24), strides=[0, 0, 128, 1])
    assert L.cp_attn_partial(r(q), r(k), r(v), 0.0, r(bcast), r(lse), None) == -10
    interleaved = _t([1, 256, 2, 128], bd.CP_F32, FAKE + (3 << 24),
                     strides=[256 * 2 * 128, 64, 128, 1])
    assert L.cp_ring_attention(r(q), r(k), r(v), (ctypes.c_int64 * 2)(0, 300), 1, 0.0,
                               r(interleaved), r(lse), None) == -10
    lse_b = _t([1, 2, 256], bd.CP_F32, FAKE + (5 << 24), strides=[512, 0, 1])
    assert L.cp_attn_partial(r(q), r(k), r(v), 0.0, r(out), r(lse_b), None) == -10
    lse2 = _t([1, 2, 256], bd.CP_F32, FAKE + (6 << 24))
    assert L.cp_lse_merge(r(bcast), r(lse), r(out), r(lse2), None) == -10
    assert L.cp_lse_merge(r(out), r(lse), r(out), r(lse2), None) == -10   # plain alias
    x = _t([2, 1, 8, 4, 128], bd.CP_BF16, FAKE)
    y = _t([2, 1, 16, 2, 128], bd.CP_BF16, FAKE + (3 << 24), strides=[0, 4096, 256, 128, 1])
    assert L.cp_ulysses_permute(r(x), r(y), 2, 0, None) == -10


def test_gathered_ring_errors():
    q, k, v, out, lse = _ok_args()
    L = bd.lib()
    r = ctypes.byref
    kg = _t([4, 1, 96, 2, 128], bd.CP_BF16, FAKE + (1 << 24))
    vg = _t([4, 1, 96, 2, 128], bd.CP_BF16, FAKE + (2 << 24))
    lens = (ctypes.c_int64 * 4)(96, 0, 50, 7)
    call = lambda lens, n, skip, acc, o=out, l=lse: L.cp_ring_attention_gathered(
        r(q), r(kg), r(vg), lens, n, skip, 0.0, acc, r(o), r(l) if l is not None else None, None)
    assert call(lens, 3, -1, 0) == -5                                   # n_chunks != slots
    assert call(lens, 4, 4, 0) == -5                                    # skip out of range
    assert call(lens, 4, -2, 0) == -5
    assert call((ctypes.c_int64 * 4)(97, 0, 50, 7), 4, -1, 0) == -5    # longer than a slot
    assert call((ctypes.c_int64 * 4)(-1, 0, 50, 7), 4, -1, 0) == -5
    assert call(None, 4, -1, 0) == -1
    bf_out = _t([1, 256, 2, 128], bd.CP_BF16, FAKE + (3 << 24))
    assert call(lens, 4, -1, 1, o=bf_out) == -2                         # accumulator is f32
    assert call(lens, 4, -1, 1, l=None) == -1                           # and needs its lse
    k4 = _t([1, 300, 2, 128], bd.CP_BF16, FAKE + (1 << 24))
    assert L.cp_ring_attention_gathered(r(q), r(k4), r(vg), lens, 4, -1, 0.0, 0, r(out),
                                        r(lse), None) == -3             # slots are 5-D


def test_partial_merge_errors():
    q, k, v, out, lse = _ok_args()
    L = bd.lib()
    r = ctypes.byref
    bf_out = _t([1, 256, 2, 128], bd.CP_BF16, FAKE + (3 << 24))
    assert L.cp_attn_partial_merge(r(q), r(k), r(v), 0.0, r(bf_out), r(lse), None) == -2
    assert L.cp_attn_partial_merge(r(q), r(k), r(v), 0.0, r(out), None, None) == -1


def test_ring_offsets_errors():
    q, k, v, out, lse = _ok_args()
    L = bd.lib()
    r = ctypes.byref

    def call(offs, n=None):
        arr = (ctypes.c_int64 * len(offs))(*offs)
        return L.cp_ring_attention(r(q), r(k), r(v), arr, len(offs) - 1 if n is None else n,
                                   0.0, r(out), r(lse), None)
    assert call([1, 300]) == -5               # must start at 0
    assert call([0, 299]) == -5               # must end at S_kv
    assert call([0, 200, 100, 300]) == -5     # monotone
    assert call([0, 300], n=0) == -5
    assert L.cp_ring_attention(r(q), r(k), r(v), None, 1, 0.0, r(out), r(lse), None) == -1


def test_permute_degree_errors():
    L = bd.lib()
    r = ctypes.byref
    x = _t([4, 1, 16, 6, 128])                 # H = 6 not divisible by 4
    y = _t([4, 1, 64, 1, 128], data=FAKE + (1 << 26))
    assert L.cp_ulysses_permute(r(x), r(y), 4, 0, None) == -6
    x = _t([3, 1, 10, 6, 64])
    y = _t([3, 1, 30, 2, 64], data=FAKE + (1 << 26))
    assert L.cp_ulysses_permute(r(x), r(y), 3, 2, None) == -3     # bad direction
    assert L.cp_ulysses_permute(r(x), r(y), 2, 0, None) == -3     # degree != shape[0]
    y16 = _t([3, 1, 30, 2, 64], bd.CP_F32, FAKE + (1 << 26))
    assert L.cp_ulysses_permute(r(x), r(y16), 3, 0, None) == -2   # dtype mismatch
    ya = _t([3, 1, 30, 2, 64], data=FAKE + 64)                     # overlaps x
    assert L.cp_ulysses_permute(r(x), r(ya), 3, 0, None) == -10


def test_merge_errors():
    L = bd.lib()
    r = ctypes.byref
    oa = _t([1, 8, 2, 128], bd.CP_F32)
    la = _t([1, 2, 8], bd.CP_F32, FAKE + (1 << 20))
    oi = _t([1, 8, 2, 128], bd.CP_BF16, FAKE + (2 << 20))
    li = _t([1, 2, 8], bd.CP_F32, FAKE + (3 << 20))
    assert L.cp_lse_merge(r(_t([1, 8, 2, 128], bd.CP_BF16)), r(la), r(oi), r(li), None) == -2
    assert L.cp_lse_merge(r(oa), r(_t([1, 2, 9], bd.CP_F32)), r(oi), r(li), None) == -3
    assert L.cp_lse_merge(r(oa), r(la), r(_t([1, 8, 2, 128], bd.CP_BF16, FAKE + 8)), r(li),
                          None) == -10


def test_usp_workspace_and_errors():
    L = bd.lib()
    # shards of 2048 tokens (a multiple of 128): permutations fold into the
    # attention kernel, no workspace
    assert L.cp_usp_workspace_bytes(2, 8192, 24, 128, bd.CP_BF16, bd.CP_F32, 2, 2) == 0
    # shards of 2050 tokens, or fp32 inputs: head-sharded q, k, v and out
    n = 2 * 8200 * 24 * 128
    assert L.cp_usp_workspace_bytes(2, 8200, 24, 128, bd.CP_BF16, bd.CP_F32, 2, 2) == 3 * n * 2 + n * 4
    n = 2 * 8192 * 24 * 128
    assert L.cp_usp_workspace_bytes(2, 8192, 24, 128, bd.CP_F32, bd.CP_F32, 2, 2) == 3 * n * 4 + n * 4
    assert L.cp_usp_workspace_bytes(2, 8192, 24, 128, 7, bd.CP_F32, 2, 2) == 0
    r = ctypes.byref
    s = lambda off, dt=bd.CP_BF16: _t([4, 2, 2050, 24, 128], dt, FAKE + off)
    q, k, v, o = s(0), s(1 << 30), s(2 << 30), s(3 << 30, bd.CP_F32)
    assert L.cp_usp_attention(r(q), r(k), r(v), 2, 2, 0.0, None, 0, r(o), None, None) == -9
    assert L.cp_usp_attention(r(q), r(k), r(v), 2, 2, 0.0, ctypes.c_void_p(FAKE), 16, r(o),
                              None, None) == -9
    assert L.cp_usp_attention(r(q), r(k), r(v), 3, 2, 0.0, None, 0, r(o), None, None) == -6


@pytest.mark.parametrize("S,R", [(256, 2), (4608, 4), (32761, 8), (5, 4), (0, 3), (7, 1)])
def test_chunk_offsets_match_generator(S, R):
    from context_attention_dits_cp_b200 import workloads as wl
    assert bd.ring_chunk_offsets(S, R) == wl.chunk_offsets(wl.ring_chunk_lengths(S, R))


def test_static_scratch_entry_rejects_oversize_before_any_launch():
    """cp_usp_attention_static refuses problems whose workspace exceeds its
    fixed array, without touching the (fake) pointers or the GPU."""
    L = bd.lib()
    r = ctypes.byref
    s = lambda off, dt=bd.CP_BF16: _t([4, 1, 2050, 24, 128], dt, FAKE + off)
    q, k, v, o = s(0), s(1 << 30), s(2 << 30), s(3 << 30, bd.CP_F32)
    need = L.cp_usp_workspace_bytes(1, 8200, 24, 128, bd.CP_BF16, bd.CP_F32, 2, 2)
    assert need > bd.USP_STATIC_SCRATCH_BYTES
    assert L.cp_usp_attention_static(r(q), r(k), r(v), 2, 2, 0.0, r(o), None, None) == -9
    assert L.cp_usp_attention_static(None, r(k), r(v), 2, 2, 0.0, r(o), None, None) == -1


def test_static_scratch_entry_reports_the_same_errors_as_the_workspace_call():
    """Argument errors come back with the codes cp_usp_attention gives,
    before the size check reads anything (all checked on the host)."""
    L = bd.lib()
    r = ctypes.byref
    s = lambda off, dt=bd.CP_BF16: _t([4, 1, 2050, 24, 128], dt, FAKE + off)
    q, k, v, o = s(0), s(1 << 30), s(2 << 30), s(3 << 30, bd.CP_F32)
    bad_dt = _t([4, 1, 2050, 24, 128], 7, FAKE + (3 << 30))
    cases = [((r(q), r(k), r(v), 3, 2, 0.0), r(o)),          # G != R * U
             ((r(q), r(k), r(v), 2, 2, 0.0), r(bad_dt)),     # unknown output dtype
             ((r(q), r(k), r(v), 0, 4, 0.0), r(o))]          # ring degree 0
    for args, out in cases:
        want = L.cp_usp_attention(*args, None, 0, out, None, None)
        assert want in (-2, -6)
        assert L.cp_usp_attention_static(*args, out, None, None) == want


def test_ulysses_anything_argument_errors():
    L = bd.lib()
    r = ctypes.byref
    B, H, D = 1, 24, 128
    so, ho = [0, 1121, 2242, 3363, 4481], [0, 6, 12, 18, 24]
    n = B * 4481 * H * D
    x, y = _t([n], data=FAKE), _t([n], data=FAKE + (1 << 30))
    off = lambda a: (ctypes.c_int64 * len(a))(*a)
    call = lambda xs, ys, s_, h_, dr=0, dg=4: L.cp_ulysses_anything_permute(
        r(xs), r(ys), B, H, D, dg, off(s_), off(h_), dr, None)
    assert call(x, y, [1, 1121, 2242, 3363, 4481], ho) == -5      # must start at 0
    assert call(x, y, [0, 1121, 1000, 3363, 4481], ho) == -5      # monotone
    assert call(x, y, so, [0, 6, 12, 18, 23]) == -5               # heads must end at H
    assert call(x, _t([n - 1], data=FAKE + (1 << 30)), so, ho) == -3
    assert call(x, _t([n], bd.CP_F32, FAKE + (1 << 30)), so, ho) == -2
    assert call(x, _t([n], data=FAKE + 64), so, ho) == -10        # overlap
    assert call(x, y, so, ho, dr=2) == -3
    assert call(x, y, so, ho, dg=0) == -6
    assert L.cp_ulysses_anything_workspace_bytes(1, 4481, 24, 128, bd.CP_BF16, bd.CP_F32) == 0
    n2 = 2 * n
    assert L.cp_ulysses_anything_workspace_bytes(2, 4481, 24, 128, bd.CP_BF16, bd.CP_F32) == \
        3 * ((n2 * 2 + 255) // 256 * 256) + (n2 * 4 + 255) // 256 * 256
    q, k, v = _t([n2], data=FAKE), _t([n2], data=FAKE + (1 << 30)), _t([n2], data=FAKE + (2 << 30))
    o = _t([n2], bd.CP_F32, FAKE + (3 << 30))
    att = lambda ws, wsb: L.cp_ulysses_anything_attention(
        r(q), r(k), r(v), 2, H, D, 4, off(so), off(ho), 0.0, ws, wsb, r(o), None, None)
    assert att(None, 0) == -9
    assert att(ctypes.c_void_p(FAKE), 1024) == -9
