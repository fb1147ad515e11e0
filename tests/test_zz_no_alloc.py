"""dash_decode_noalloc: the decode step for callers that cannot obtain device memory of their
own (a plugin inside a runtime that owns every device allocation, a service that must not grow
its footprint).  It takes no workspace; its scratch is a fixed 16 MiB array inside the library.

The GPU test calls it through the C ABI.  A first call on a different shape leaves unrelated
values in the shared array; then two decode steps in a row must equal dash_decode (the workspace
version, same kernels) bit for bit, and the status word each call returns must be 0.  This file
is collected last on purpose, so a run that stops at the first failure has run the others.
"""
import ctypes

import pytest
import torch

import adaptive_sparse_hierarchical_b200 as D
from adaptive_sparse_hierarchical_b200 import _lib as L
from adaptive_sparse_hierarchical_b200 import inputs


def _noalloc():
    f = L.load().dash_decode_noalloc
    f.argtypes = [ctypes.POINTER(L.dash_params)] + [ctypes.c_void_p] * 8
    f.restype = ctypes.c_int
    return f


def test_oversize_request_is_rejected():
    """The full-size decode shape needs ~37 MB of scratch: rejected before anything runs."""
    st = (132096 * 2 * 128, 2 * 128, 128)
    p = L.params(batch=8, seqlen=132096, h_q=32, h_kv=2, d_h=128, chunk=64, alpha=1.5, gamma=4.0,
                 k_strides=st, v_strides=st)
    assert L.dash_workspace_size(p, L.DASH_OP_DECODE) > 16 << 20
    assert _noalloc()(ctypes.byref(p), 256, 256, 256, 256, 256, 256, None, None) == L.DASH_EWORKSPACE


def test_invalid_params_are_rejected_like_dash_decode():
    st = (2048 * 2 * 128, 2 * 128, 128)
    p = L.params(batch=1, seqlen=2048, h_q=16, h_kv=2, d_h=96, chunk=64, alpha=1.5, gamma=4.0,
                 k_strides=st, v_strides=st)
    assert _noalloc()(ctypes.byref(p), 256, 256, 256, 256, 256, 256, None, None) == L.DASH_EUNSUPPORTED
    p.d_h, p.alpha = 128, 2.5
    assert _noalloc()(ctypes.byref(p), 256, 256, 256, 256, 256, 256, None, None) == L.DASH_EINVAL


def _state(seed, b, cap, hq, hkv, prefix, gamma):
    d, B = 128, 64
    x = inputs.planted(seed, b, cap, hq, hkv, d, B, dtype="bf16", chunk_frac=0.1)
    dev = {k: torch.from_numpy(x[k]).to("cuda", torch.bfloat16) for k in ("Q", "K", "V")}
    st = D.DecodeState(b, cap, hq, hkv, d, chunk=B, alpha=1.5, gamma=gamma,
                       qbar=torch.from_numpy(x["qbar"]).cuda())
    st.fill(dev["K"][:, :max(prefix)], dev["V"][:, :max(prefix)], prefix)
    return st, dev


def _call(f, st, q, out, status, stream):
    return f(ctypes.byref(st.p), q.data_ptr(), st.K.data_ptr(), st.V.data_ptr(), st.kbar.data_ptr(),
             st.seqlens.data_ptr(), out.data_ptr(), status.data_ptr(), stream)


@pytest.mark.gpu
def test_noalloc_decode_equals_workspace_decode_two_calls():
    f = _noalloc()
    stream = torch.cuda.current_stream().cuda_stream
    status = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    # another shape first (batch, capacity, heads and lengths differ): its values stay in the array
    other, odev = _state(17, 2, 1024, 8, 2, [900, 333], 5.0)
    q0 = odev["Q"][torch.arange(2), other.seqlens.long().cpu() - 1].contiguous()
    junk = torch.empty_like(q0)
    assert _call(f, other, q0, junk, status, stream) == L.DASH_OK
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    del other, odev

    b = 3
    st, dev = _state(31, b, 2048, 16, 2, [1500, 777, 64], 6.0)
    rows = torch.arange(b)
    for _ in range(2):
        pos = st.seqlens.long().cpu()
        st.append(dev["K"][rows, pos].contiguous(), dev["V"][rows, pos].contiguous())
        q = dev["Q"][rows, pos].contiguous()
        ref = st.decode(q).clone()
        torch.cuda.synchronize()
        assert st.workspace[L.dash_error_word_offset(st.p, L.DASH_OP_DECODE):][:4].view(torch.int32).item() == 0
        out = torch.full_like(ref, float("nan"))
        status.fill_(-7)
        rc = _call(f, st, q, out, status, stream)
        assert rc == L.DASH_OK, L.dash_status_string(rc)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(out, ref)
