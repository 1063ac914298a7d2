"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/loopvq.h declares, and validates arguments on the
host (all calls here return before any CUDA launch)."""
import os
import re

import pytest

from sub_bit_vector_b200 import loopvq as L

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "loopvq.h")
FAKE = 1 << 20          # a 256-byte-aligned non-null address; never dereferenced on these paths


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"LOOPVQ_API\s+[\w\s\*]+?\b(loopvq_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported_and_bound():
    names = _declared()
    assert len(names) >= 17
    for n in names:
        assert hasattr(L._lib, n), n
        assert n in L.EXPORTED, n
        assert callable(getattr(L, n)), n


def test_library_keeps_no_encode_fault_word():
    """Encode faults go to a word the caller passes; the library exports no
    reader of a global one (its only global state is the allocation-free
    decode's scratch array)."""
    assert not hasattr(L._lib, "loopvq_read_encode_faults")
    assert "loopvq_read_encode_faults" not in open(HEADER).read()


def test_version_and_status_strings():
    assert "sm_100a" in L.loopvq_version()
    for s in range(6):
        assert L.loopvq_status_string(s) != "unknown status"
    assert L.loopvq_status_string(99) == "unknown status"


def test_bits_and_sizes():
    d = L.make_desc(4, 4, 16, 128, 16)
    assert L.loopvq_validate_desc(d) == L.LOOPVQ_OK
    assert L.loopvq_bits_per_element(d) == 0.5
    assert L.loopvq_bits_per_element(L.make_desc(4, 4, 16, 128, 32)) == 0.25
    # canonical 1*16*32*256*16 bf16 = 4 MiB, then 4 step slices of 1 MiB
    assert L.loopvq_codebook_packed_bytes(d) == 4 * 2**20 + 4 * 2**20
    assert L.loopvq_index_pool_bytes(d, 32768) == 16 * 32768 * 32
    assert L.loopvq_index_pool_bytes(d, 100) == 0
    assert L.loopvq_ctx_split(32768, 64, 256, 8) == (64, 32448, 256)
    assert L.loopvq_ctx_split(10, 64, 256, 8) == (10, 0, 0)
    with pytest.raises(L.LoopVQError):
        L.loopvq_ctx_split(-1, 64, 256, 8)


@pytest.mark.parametrize("args,status", [
    ((4, 3, 16, 128, 16), L.LOOPVQ_ERR_INVALID_ARG),     # Tc does not divide T
    ((4, 4, 16, 128, 18), L.LOOPVQ_ERR_INVALID_ARG),     # G not a multiple of Tc
    ((4, 4, 16, 102, 16), L.LOOPVQ_ERR_INVALID_ARG),     # D not a multiple of W
    ((4, 4, 16, 128, 8), L.LOOPVQ_ERR_UNSUPPORTED),      # W=2 -> J=64
    ((4, 4, 16, 256, 16), L.LOOPVQ_ERR_UNSUPPORTED),     # J=64
    ((4, 4, 16, 96, 16), L.LOOPVQ_ERR_UNSUPPORTED),      # J=24
])
def test_descriptor_validation(args, status):
    assert L.loopvq_validate_desc(L.make_desc(*args)) == status


def test_codes_count_bounds():
    assert L.loopvq_validate_desc(L.make_desc(4, 4, 16, 128, 16, n_codes=0)) == L.LOOPVQ_ERR_INVALID_ARG
    assert L.loopvq_validate_desc(L.make_desc(4, 4, 16, 128, 16, n_codes=257)) == L.LOOPVQ_ERR_INVALID_ARG
    assert L.loopvq_validate_desc(L.make_desc(4, 4, 16, 128, 16, n_codes=7)) == L.LOOPVQ_OK
    assert L.loopvq_validate_desc(L.make_desc(4, 4, 4, 128, 16, n_heads_q=6)) == L.LOOPVQ_ERR_INVALID_ARG


def _layout(**kw):
    a = dict(batch=1, n_sink=64, n_recent=256, page=8, max_ctx_len=32768, ctx_len=FAKE, body_off=FAKE,
             win_off=FAKE, body_pool_tokens=32768, win_pool_tokens=320)
    a.update(kw)
    return L.make_layout(**a)


def test_workspace_sizes():
    d = L.make_desc(4, 4, 16, 128, 16)
    ws = L.loopvq_decode_workspace_bytes(d, _layout())
    assert ws > 256 and ws % 4 == 0
    assert L.loopvq_decode_workspace_bytes(d, _layout(body_pool_tokens=33)) == 0
    assert L.loopvq_decode_workspace_bytes(d, _layout(batch=0)) == 0
    assert L.loopvq_dense_decode_workspace_bytes(1, 16, 128, 32768) > 256


def _decode(d, layout, **kw):
    a = dict(cbK=FAKE, cbV=FAKE, idxK=FAKE, idxV=FAKE, winK=FAKE, winV=FAKE, q=FAKE, qd=L.LOOPVQ_BF16, t=0,
             out=FAKE, od=L.LOOPVQ_F32, lse=None, ws=FAKE, wsb=1 << 30)
    a.update(kw)
    return L._lib.loopvq_decode_attn(d, a["cbK"], a["cbV"], layout, a["idxK"], a["idxV"], a["winK"], a["winV"],
                                     a["q"], a["qd"], a["t"], 0.088, a["out"], a["od"], a["lse"], a["ws"],
                                     a["wsb"], None)


def test_decode_rejects_bad_arguments_before_launch():
    d = L.make_desc(4, 4, 16, 128, 16)
    lay = _layout()
    import ctypes
    D, Lp = ctypes.byref(d), ctypes.byref(lay)
    assert _decode(D, Lp, t=4) == L.LOOPVQ_ERR_INVALID_ARG
    assert _decode(D, Lp, t=-1) == L.LOOPVQ_ERR_INVALID_ARG
    assert _decode(D, Lp, idxK=FAKE + 8) == L.LOOPVQ_ERR_INVALID_ARG
    assert _decode(D, Lp, ws=FAKE + 16) == L.LOOPVQ_ERR_INVALID_ARG
    assert _decode(D, Lp, q=None) == L.LOOPVQ_ERR_INVALID_ARG
    assert _decode(D, Lp, qd=7) == L.LOOPVQ_ERR_INVALID_ARG
    assert _decode(D, Lp, wsb=128) == L.LOOPVQ_ERR_WORKSPACE_TOO_SMALL
    bad = L.make_desc(4, 4, 16, 128, 8)
    assert _decode(ctypes.byref(bad), Lp) == L.LOOPVQ_ERR_UNSUPPORTED
    lay2 = _layout(ctx_len=None)
    assert _decode(D, ctypes.byref(lay2)) == L.LOOPVQ_ERR_INVALID_ARG


def test_encode_and_pool_reject_bad_arguments():
    import ctypes
    d = L.make_desc(4, 4, 16, 128, 16)
    D = ctypes.byref(d)
    enc = L._lib.loopvq_encode
    assert enc(D, FAKE, 0, FAKE, 1, 8, 1, 1, 1, FAKE, 30, 32, None, None) == L.LOOPVQ_ERR_INVALID_ARG  # past pool end
    assert enc(D, FAKE, 2, FAKE, 1, 8, 1, 1, 1, FAKE, 0, 32, None, None) == L.LOOPVQ_ERR_INVALID_ARG   # bad kind
    assert enc(D, FAKE, 0, FAKE, 3, 8, 1, 1, 1, FAKE, 0, 32, None, None) == L.LOOPVQ_ERR_INVALID_ARG   # bad dtype
    assert enc(D, FAKE, 0, FAKE, 1, 8, -1, 1, 1, FAKE, 0, 32, None, None) == L.LOOPVQ_ERR_INVALID_ARG  # stride
    assert enc(D, FAKE + 4, 0, FAKE, 1, 8, 1, 1, 1, FAKE, 0, 32, None, None) == L.LOOPVQ_ERR_INVALID_ARG  # align
    assert enc(D, FAKE, 0, FAKE, 1, 0, 1, 1, 1, FAKE, 0, 32, None, None) == L.LOOPVQ_OK           # empty
    # the fault word is the caller's: a misaligned one is refused before any launch
    assert enc(D, FAKE, 0, FAKE, 1, 8, 1, 1, 1, FAKE, 0, 32, FAKE + 2, None) == L.LOOPVQ_ERR_INVALID_ARG
    assert enc(D, FAKE, 0, FAKE, 1, 0, 1, 1, 1, FAKE, 0, 32, FAKE, None) == L.LOOPVQ_OK
    pack = L._lib.loopvq_index_pool_pack
    assert pack(D, 0, FAKE, 10, FAKE, 30, 32, None) == L.LOOPVQ_ERR_INVALID_ARG
    assert pack(D, 0, FAKE, 10, FAKE, 0, 33, None) == L.LOOPVQ_ERR_INVALID_ARG
    assert pack(D, 0, FAKE, 0, FAKE, 0, 32, None) == L.LOOPVQ_OK
    cbp = L._lib.loopvq_codebook_pack
    assert cbp(D, FAKE, FAKE + 8, 1 << 30, None) == L.LOOPVQ_ERR_INVALID_ARG
    assert cbp(D, FAKE, FAKE * 64, 16, None) == L.LOOPVQ_ERR_INVALID_ARG
    assert cbp(D, FAKE, FAKE + 256, 1 << 30, None) == L.LOOPVQ_ERR_INVALID_ARG   # overlapping buffers


def test_dense_rejects_bad_arguments():
    dd = L._lib.loopvq_dense_decode_attn
    assert dd(1, 16, 16, 96, 100, FAKE, FAKE, 100, FAKE, FAKE, FAKE, 1, 0.1, FAKE, None, FAKE, 1 << 30,
              None) == L.LOOPVQ_ERR_UNSUPPORTED
    assert dd(1, 16, 24, 128, 100, FAKE, FAKE, 100, FAKE, FAKE, FAKE, 1, 0.1, FAKE, None, FAKE, 1 << 30,
              None) == L.LOOPVQ_ERR_INVALID_ARG
    assert dd(1, 16, 16, 128, 100, FAKE, FAKE, 100, FAKE, FAKE, FAKE, 1, 0.1, FAKE, None, FAKE, 64,
              None) == L.LOOPVQ_ERR_WORKSPACE_TOO_SMALL


def test_paged_ring_and_new_token_layout_validation():
    """Paged body, ring window and current-token inputs are validated on the
    host: an invalid combination gives a zero workspace size."""
    d = L.make_desc(4, 4, 16, 128, 16)
    P, R, NT = L.LOOPVQ_LAYOUT_PAGED_BODY, L.LOOPVQ_LAYOUT_RING_WINDOW, L.LOOPVQ_LAYOUT_STATIC_INPUTS
    paged = dict(flags=P, body_pages=FAKE, body_page_tokens=256, max_body_pages=127, body_off=None)
    assert L.loopvq_decode_workspace_bytes(d, _layout(**paged)) > 0          # body_off unused when paged
    assert L.loopvq_decode_workspace_bytes(d, _layout(**dict(paged, max_body_pages=126))) == 0   # too few pages
    assert L.loopvq_decode_workspace_bytes(d, _layout(**dict(paged, body_page_tokens=48))) == 0  # not a multiple of 32
    assert L.loopvq_decode_workspace_bytes(d, _layout(**dict(paged, body_page_tokens=36))) == 0
    assert L.loopvq_decode_workspace_bytes(d, _layout(**dict(paged, body_pages=None))) == 0
    assert L.loopvq_decode_workspace_bytes(d, _layout(body_off=None)) == 0    # contiguous body needs body_off
    ring = dict(flags=R | NT, win_head=FAKE, win_ring=264)
    assert L.loopvq_decode_workspace_bytes(d, _layout(**ring)) > 0
    assert L.loopvq_decode_workspace_bytes(d, _layout(**dict(ring, win_ring=262))) == 0        # < n_recent + page - 1
    assert L.loopvq_decode_workspace_bytes(d, _layout(**dict(ring, win_head=None))) == 0
    assert L.loopvq_decode_workspace_bytes(d, _layout(flags=0x80)) == 0                         # unknown flag
    assert L.loopvq_decode_workspace_bytes(d, _layout(new_k=FAKE, new_v=FAKE)) > 0
    assert L.loopvq_decode_workspace_bytes(d, _layout(new_k=FAKE)) == 0                         # K without V
    assert L.loopvq_decode_workspace_bytes(d, _layout(new_k=FAKE + 2, new_v=FAKE)) == 0         # misaligned


def test_codebook_grad_rejects_bad_arguments_before_launch():
    import ctypes
    d = L.make_desc(4, 4, 16, 128, 16)
    lay = _layout()
    D, Lp = ctypes.byref(d), ctypes.byref(lay)
    fn = L._lib.loopvq_codebook_grad

    def call(desc=D, layout=Lp, idxK=FAKE, q=FAKE, qd=L.LOOPVQ_BF16, t=0, lse=FAKE, target=FAKE, gk=FAKE,
             weight=1.0):
        return fn(desc, FAKE, FAKE, layout, idxK, FAKE, q, qd, t, 0.088, FAKE, lse, target, weight, gk, FAKE, None,
                  None, None)
    assert call(t=4) == L.LOOPVQ_ERR_INVALID_ARG
    assert call(t=-1) == L.LOOPVQ_ERR_INVALID_ARG
    assert call(idxK=FAKE + 8) == L.LOOPVQ_ERR_INVALID_ARG
    assert call(q=None) == L.LOOPVQ_ERR_INVALID_ARG
    assert call(lse=None) == L.LOOPVQ_ERR_INVALID_ARG
    assert call(target=None) == L.LOOPVQ_ERR_INVALID_ARG
    assert call(gk=None) == L.LOOPVQ_ERR_INVALID_ARG
    assert call(qd=7) == L.LOOPVQ_ERR_INVALID_ARG
    assert call(weight=float("nan")) == L.LOOPVQ_ERR_INVALID_ARG
    bad = L.make_desc(4, 4, 16, 128, 8)     # J = 64
    assert call(desc=ctypes.byref(bad)) == L.LOOPVQ_ERR_UNSUPPORTED
    lay2 = _layout(ctx_len=None)
    assert call(layout=ctypes.byref(lay2)) == L.LOOPVQ_ERR_INVALID_ARG


def test_decode_steps_rejects_bad_step_ranges():
    import ctypes
    d = L.make_desc(4, 2, 16, 128, 8)
    lay = _layout()
    D, Lp = ctypes.byref(d), ctypes.byref(lay)
    assert L._lib.loopvq_decode_steps_workspace_bytes(D, Lp, 4) >= L._lib.loopvq_decode_steps_workspace_bytes(D, Lp, 1)
    assert L._lib.loopvq_decode_steps_workspace_bytes(D, Lp, 1) == L._lib.loopvq_decode_workspace_bytes(D, Lp)
    assert L._lib.loopvq_decode_steps_workspace_bytes(D, Lp, 5) == 0
    assert L._lib.loopvq_decode_steps_workspace_bytes(D, Lp, 0) == 0
    fn = L._lib.loopvq_decode_attn_steps

    def call(first, n, wsb=1 << 30):
        return fn(D, FAKE, FAKE, Lp, FAKE, FAKE, FAKE, FAKE, FAKE, L.LOOPVQ_BF16, first, n, 0.088, FAKE, L.LOOPVQ_F32,
                  None, FAKE, wsb, None)
    assert call(0, 0) == L.LOOPVQ_ERR_INVALID_ARG
    assert call(2, 3) == L.LOOPVQ_ERR_INVALID_ARG
    assert call(-1, 2) == L.LOOPVQ_ERR_INVALID_ARG
    assert call(1, 2, wsb=256) == L.LOOPVQ_ERR_WORKSPACE_TOO_SMALL


def test_residual_sizes_and_argument_errors():
    import ctypes
    d = L.make_residual_desc(4, 2, 128, n_heads_q=4)
    D = ctypes.byref(d)
    assert L.loopvq_residual_codes_bytes(d, 64) == 4 * 2 * 64 * 64
    assert L.loopvq_residual_params_bytes(d, L.LOOPVQ_KEYS, 64) == 4 * 2 * 2 * 128 * 4
    assert L.loopvq_residual_params_bytes(d, L.LOOPVQ_VALUES, 64) == 4 * 2 * 64 * 4 * 4
    assert L.loopvq_residual_codes_bytes(d, 48) == 0
    bad = L.make_residual_desc(4, 2, 96)
    assert L._lib.loopvq_residual_codes_bytes(ctypes.byref(bad), 64) == 0
    enc = L._lib.loopvq_residual_encode
    assert enc(D, 0, FAKE, 0, 10, 1, 1, 1, FAKE, FAKE, 16, 64, None) == L.LOOPVQ_ERR_INVALID_ARG   # unaligned offset
    assert enc(D, 0, FAKE, 0, 40, 1, 1, 1, FAKE, FAKE, 32, 64, None) == L.LOOPVQ_ERR_INVALID_ARG   # past pool end
    assert enc(D, 2, FAKE, 0, 10, 1, 1, 1, FAKE, FAKE, 0, 64, None) == L.LOOPVQ_ERR_INVALID_ARG    # bad kind
    assert enc(ctypes.byref(bad), 0, FAKE, 0, 10, 1, 1, 1, FAKE, FAKE, 0, 64, None) == L.LOOPVQ_ERR_UNSUPPORTED
    assert enc(D, 0, FAKE, 0, 0, 1, 1, 1, FAKE, FAKE, 0, 64, None) == L.LOOPVQ_OK                 # empty
    dec = L._lib.loopvq_residual_decode_attn
    ws = L.loopvq_residual_decode_workspace_bytes(d, 2, 1000)
    assert ws > 0

    def call(t=0, q=FAKE, wsb=ws, pool=64):
        return dec(D, 2, 1000, FAKE, FAKE, pool, FAKE, FAKE, FAKE, FAKE, q, L.LOOPVQ_BF16, t, 0.088, FAKE, None, FAKE,
                   wsb, None)
    assert call(t=4) == L.LOOPVQ_ERR_INVALID_ARG
    assert call(q=None) == L.LOOPVQ_ERR_INVALID_ARG
    assert call(pool=40) == L.LOOPVQ_ERR_INVALID_ARG
    assert call(wsb=256) == L.LOOPVQ_ERR_WORKSPACE_TOO_SMALL
