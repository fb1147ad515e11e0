"""CPU checks of the C-ABI library: it loads, exports every entry point include/dash.h declares,
and rejects bad arguments before launching anything (no GPU needed for these paths)."""
import ctypes
import subprocess

import pytest

import adaptive_sparse_hierarchical_b200 as D
from adaptive_sparse_hierarchical_b200 import _lib as L
from adaptive_sparse_hierarchical_b200.build import LIB, build


@pytest.fixture(scope="module", autouse=True)
def _built():
    build()


def _p(**kw):
    base = dict(batch=1, seqlen=1024, h_q=8, h_kv=2, d_h=128, chunk=64, alpha=1.5, gamma=8.0, dtype=L.DASH_BF16,
                q_strides=(1024 * 8 * 128, 8 * 128, 128), k_strides=(1024 * 2 * 128, 256, 128),
                v_strides=(1024 * 2 * 128, 256, 128), o_strides=(1024 * 8 * 128, 8 * 128, 128))
    base.update(kw)
    return L.params(**base)


def test_header_symbols_exported():
    syms = L.header_symbols()
    assert set(syms) == {"dash_workspace_size", "dash_route_capacity", "dash_prefill", "dash_prefill_stage",
                         "dash_summary_build", "dash_error_word_offset", "dash_decode_noalloc", "dash_prefill_order_offset",
                         "dash_summary_append", "dash_decode", "dash_status_string", "dash_summary_build_paged",
                         "dash_summary_append_paged", "dash_decode_paged", "dash_backward", "dash_set_wait_limit"}
    lib = D.load()
    for s in syms:
        assert hasattr(lib, s), s
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(syms) <= exported


def test_route_capacity_is_triangular_sum():
    for n, B in [(1, 64), (63, 64), (64, 64), (65, 64), (1000, 32), (32768, 64), (5, 16)]:
        p = _p(seqlen=n, chunk=B)
        assert L.dash_route_capacity(p) == sum(i // B for i in range(n))


def test_workspace_sizes_cover_layout():
    p = _p()
    T, cap = 1024 // 64, L.dash_route_capacity(_p())
    need = 2 * T * 128 * 4 + 2 * 1024 * 4 + 2 * 2 * cap * 4
    assert L.dash_workspace_size(p, L.DASH_OP_PREFILL) >= need
    assert L.dash_workspace_size(p, L.DASH_OP_DECODE) > 0
    assert L.dash_workspace_size(p, 7) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(h_q=6, h_kv=4), L.DASH_EINVAL),
    (dict(alpha=1.0), L.DASH_EINVAL),
    (dict(alpha=2.5), L.DASH_EINVAL),
    (dict(gamma=-1.0), L.DASH_EINVAL),
    (dict(inv_sigma=-0.5), L.DASH_EINVAL),
    (dict(batch=0), L.DASH_EINVAL),
    (dict(dtype=7), L.DASH_EINVAL),
    (dict(d_h=96), L.DASH_EUNSUPPORTED),
    (dict(chunk=48), L.DASH_EUNSUPPORTED),
    (dict(h_q=6, h_kv=2), L.DASH_EUNSUPPORTED),
    (dict(h_q=64, h_kv=2), L.DASH_EUNSUPPORTED),
])
def test_bad_params_rejected_before_launch(kw, code):
    assert L.dash_prefill(_p(**kw), 256, 256, 256, 256, 256, workspace=256, ws_bytes=1 << 40, check=False) == code
    assert L.dash_workspace_size(_p(**kw), L.DASH_OP_PREFILL) == 0


def test_missing_pointers_workspace_and_alignment():
    p = _p()
    ws = L.dash_workspace_size(p, L.DASH_OP_PREFILL)
    assert L.dash_prefill(p, 0, 256, 256, 256, 256, workspace=256, ws_bytes=ws, check=False) == L.DASH_EINVAL
    assert L.dash_prefill(p, 256, 256, 256, 256, 256, check=False) == L.DASH_EWORKSPACE
    assert L.dash_prefill(p, 256, 256, 256, 256, 256, workspace=256, ws_bytes=ws - 1, check=False) == L.DASH_EWORKSPACE
    assert L.dash_prefill(p, 264, 256, 256, 256, 256, workspace=256, ws_bytes=ws, check=False) == L.DASH_EALIGN
    assert L.dash_prefill(p, 256, 256, 256, 256, 256, workspace=384, ws_bytes=ws, check=False) == L.DASH_EALIGN
    bad = _p(k_strides=(1024 * 2 * 128, 250, 128))
    assert L.dash_prefill(bad, 256, 256, 256, 256, 256, workspace=256, ws_bytes=ws, check=False) == L.DASH_EALIGN


def test_status_strings():
    for rc in (0, -1, -2, -3, -4, -5, -99):
        assert isinstance(L.dash_status_string(rc), str) and L.dash_status_string(rc)


@pytest.mark.parametrize("kw,pkw,code", [
    (dict(), dict(page_size=96), L.DASH_EUNSUPPORTED),        # not a multiple of 64
    (dict(chunk=128), dict(page_size=64), L.DASH_EUNSUPPORTED),   # a chunk would straddle two pages
    (dict(), dict(max_pages=7), L.DASH_EINVAL),               # 7 * 128 < seqlen 1024
    (dict(), dict(page_size=0), L.DASH_EINVAL),
    (dict(), dict(num_pages=0), L.DASH_EINVAL),
    (dict(), dict(page_table=0), L.DASH_EINVAL),
    (dict(d_h=64, q_strides=(1024 * 8 * 64, 8 * 64, 64), k_strides=(1024 * 2 * 64, 128, 64),
          v_strides=(1024 * 2 * 64, 128, 64), o_strides=(1024 * 8 * 64, 8 * 64, 64)), dict(), L.DASH_EUNSUPPORTED),
    (dict(dtype=L.DASH_F32), dict(), L.DASH_EUNSUPPORTED),
    (dict(), dict(k_page_stride=128 * 256 + 4), L.DASH_EALIGN),   # pages 8 bytes apart from a 16-byte boundary
])
def test_paged_description_rejected_before_launch(kw, pkw, code):
    """The paged entry points check the page description before touching the device."""
    base = dict(page_table=256, max_pages=8, page_size=128, num_pages=64, k_page_stride=128 * 256,
                v_page_stride=128 * 256)
    base.update(pkw)
    pk = L.dash_paged_kv(base["page_table"], base["max_pages"], base["page_size"], base["num_pages"],
                         base["k_page_stride"], base["v_page_stride"])
    p = _p(**kw)
    lib = D.load()
    assert lib.dash_decode_paged(ctypes.byref(p), ctypes.byref(pk), 256, 256, 256, 256, 256, 256, None, 256,
                                 1 << 40, None) == code
    assert lib.dash_summary_build_paged(ctypes.byref(p), ctypes.byref(pk), 256, 256, 256, 256, 256, None) == code
    assert lib.dash_summary_append_paged(ctypes.byref(p), ctypes.byref(pk), 256, 256, 256, 256, 256, 256, 256,
                                         256, None) == code
    # a null page description is an error, not the contiguous layout
    assert lib.dash_decode_paged(ctypes.byref(_p()), None, 256, 256, 256, 256, 256, 256, None, 256, 1 << 40,
                                 None) == L.DASH_EINVAL


def test_backward_arguments_rejected_before_launch():
    """dash_backward checks its arguments before touching the device: the route lists are
    required, the workspace must cover dash_workspace_size(p, DASH_OP_BACKWARD), and a group whose
    chunk logits do not fit the query-major kernel's shared memory is unsupported."""
    lib = D.load()
    p = _p()
    ws = L.dash_workspace_size(p, L.DASH_OP_BACKWARD)
    T, cap, g = 1024 // 64, L.dash_route_capacity(p), 4
    assert ws >= 2 * 8 * 1024 * 4 + 2 * cap * g * 4 + 2 * 2 * cap * 4 + 2 * 2 * T * 128 * 4
    full = L.dash_route_out(256, 256, 256, None)
    no_bias = L.dash_route_out(256, 256, None, None)

    def call(pp, route, workspace=256, nbytes=ws):
        return lib.dash_backward(ctypes.byref(pp), 256, 256, 256, 256, 256, 256,
                                 ctypes.byref(route) if route is not None else None, 256, 256, 256, 256,
                                 workspace, nbytes, None)

    assert call(p, None) == L.DASH_EINVAL
    assert call(p, no_bias) == L.DASH_EINVAL
    assert call(p, full, workspace=None) == L.DASH_EWORKSPACE
    assert call(p, full, nbytes=ws - 1) == L.DASH_EWORKSPACE
    assert call(p, full, workspace=384) == L.DASH_EALIGN
    assert call(_p(alpha=1.0), full) == L.DASH_EINVAL
    # 16 heads per group x 4096 chunks of logits (plus the per-entry buffers) exceed shared memory
    big = _p(seqlen=131072, h_q=32, h_kv=2, chunk=32, q_strides=(0, 32 * 128, 128), k_strides=(0, 256, 128),
             v_strides=(0, 256, 128), o_strides=(0, 32 * 128, 128))
    assert call(big, full, nbytes=1 << 50) == L.DASH_EUNSUPPORTED


def test_wait_limit_knob_round_trips():
    """The diagnostic poll limit: the previous value comes back, a negative one is refused."""
    prev = L.dash_set_wait_limit(5)
    assert prev == 1 << 23
    assert L.dash_set_wait_limit(-1) == -1
    assert L.dash_set_wait_limit(prev) == 5


def test_prefill_order_offset_rejects_invalid_params():
    """The diagnostic offset of Stage 2's position order: -1 for invalid params and for shapes whose
    tensor-core Stage 2 keeps sequence order (g = 2); otherwise it lies inside the workspace."""
    assert L.dash_prefill_order_offset(_p(h_q=6, h_kv=4)) == -1
    assert L.dash_prefill_order_offset(_p(alpha=1.0)) == -1
    assert L.dash_prefill_order_offset(_p(h_q=4, h_kv=2)) == -1
    p = _p()
    off = L.dash_prefill_order_offset(p)
    assert off == -1 or 0 <= off < L.dash_workspace_size(p, L.DASH_OP_PREFILL)
