"""dash_decode_noalloc: the decode step for callers that cannot obtain device memory of their
own (a plugin inside a runtime that owns every device allocation, a service that must not grow
its footprint).  It takes no workspace; its scratch is a fixed 16 MiB array inside the library.

The GPU test calls it through the C ABI on two decode steps in a row and checks each output
against dash_decode (the workspace version) on the same caches, within the bf16 tolerance of
the parity tests.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import adaptive_sparse_hierarchical_b200 as D
from adaptive_sparse_hierarchical_b200 import _lib as L
from adaptive_sparse_hierarchical_b200 import inputs


def _noalloc():
    f = L.load().dash_decode_noalloc
    f.argtypes = [ctypes.POINTER(L.dash_params)] + [ctypes.c_void_p] * 7
    f.restype = ctypes.c_int
    return f


def test_oversize_request_is_rejected():
    """The full-size decode shape needs ~37 MB of scratch: rejected before anything runs."""
    st = (132096 * 2 * 128, 2 * 128, 128)
    p = L.params(batch=8, seqlen=132096, h_q=32, h_kv=2, d_h=128, chunk=64, alpha=1.5, gamma=4.0,
                 k_strides=st, v_strides=st)
    assert _noalloc()(ctypes.byref(p), 256, 256, 256, 256, 256, 256, None) == L.DASH_EWORKSPACE


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_decode_two_calls():
    b, cap, hq, hkv, d, B = 3, 2048, 16, 2, 128, 64
    x = inputs.planted(31, b, cap, hq, hkv, d, B, dtype="bf16", chunk_frac=0.1)
    dev = {k: torch.from_numpy(x[k]).to("cuda", torch.bfloat16) for k in ("Q", "K", "V")}
    st = D.DecodeState(b, cap, hq, hkv, d, chunk=B, alpha=1.5, gamma=6.0, qbar=torch.from_numpy(x["qbar"]).cuda())
    lengths = [1500, 777, 64]
    st.fill(dev["K"][:, :1500], dev["V"][:, :1500], lengths)
    f = _noalloc()
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        pos = st.seqlens.long().cpu()
        rows = torch.arange(b)
        st.append(dev["K"][rows, pos].contiguous(), dev["V"][rows, pos].contiguous())
        q = dev["Q"][rows, pos].contiguous()
        ref = st.decode(q).clone()
        out = torch.full_like(ref, float("nan"))
        rc = f(ctypes.byref(st.p), q.data_ptr(), st.K.data_ptr(), st.V.data_ptr(), st.kbar.data_ptr(),
               st.seqlens.data_ptr(), out.data_ptr(), stream)
        assert rc == L.DASH_OK, L.dash_status_string(rc)
        torch.cuda.synchronize()
        err = (out.float() - ref.float()).abs()
        assert torch.isfinite(out.float()).all()
        assert err.max().item() <= 2e-2 and (err.mean() / ref.float().abs().mean()).item() <= 1e-2
