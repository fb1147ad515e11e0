"""Tensor-level helpers over the C ABI: allocate outputs / workspace with torch and call the
library.  All arithmetic happens in the CUDA kernels of libdash_b200.so."""
from __future__ import annotations

import torch

from . import _lib as L


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return L.DASH_BF16
    if t.dtype == torch.float32:
        return L.DASH_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _st(t: torch.Tensor):
    """Element strides {batch, position, head} of a [b, n, h, d] tensor with d contiguous."""
    assert t.dim() == 4 and t.stride(3) == 1, "head dimension must be contiguous"
    return (t.stride(0), t.stride(1), t.stride(2))


def prefill_params(Q, K, V, O, *, chunk, alpha, gamma, inv_sigma=1.0):
    b, n, hq, d = Q.shape
    return L.params(batch=b, seqlen=n, h_q=hq, h_kv=K.shape[2], d_h=d, chunk=chunk, alpha=alpha, gamma=gamma,
                    inv_sigma=inv_sigma, dtype=_dtype_code(Q), q_strides=_st(Q), k_strides=_st(K),
                    v_strides=_st(V), o_strides=_st(O))


class Prefill:
    """Reusable causal prefill call: buffers are allocated once for a fixed shape."""

    def __init__(self, Q, K, V, qbar, *, chunk, alpha, gamma, inv_sigma=1.0, want_route=False, bitmask=False,
                 O=None):
        self.Q, self.K, self.V, self.qbar = Q, K, V, qbar
        self.O = torch.empty_like(Q) if O is None else O
        self.p = prefill_params(Q, K, V, self.O, chunk=chunk, alpha=alpha, gamma=gamma, inv_sigma=inv_sigma)
        dev = Q.device
        b, n, hq, d = Q.shape
        hkv = K.shape[2]
        T = n // chunk
        self.kbar = torch.empty((b, hkv, T, d), dtype=torch.float32, device=dev)
        self.route = None
        self.counts = self.chunk_idx = self.bias = self.bitmask = None
        if want_route:
            cap = L.dash_route_capacity(self.p)
            self.counts = torch.empty((b, hkv, n), dtype=torch.int32, device=dev)
            self.chunk_idx = torch.empty((b, hkv, max(cap, 1)), dtype=torch.int32, device=dev)
            self.bias = torch.empty((b, hkv, max(cap, 1)), dtype=torch.float32, device=dev)
            if bitmask:
                self.bitmask = torch.empty((b, hkv, n, (T + 31) // 32), dtype=torch.int32, device=dev)
            self.route = L.route_out(self.counts, self.chunk_idx, self.bias, self.bitmask)
        ws = L.dash_workspace_size(self.p, L.DASH_OP_PREFILL)
        self.workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)

    def stage(self, k, stream=None):
        """Run one stage (0, 1 or 2) alone on the stored buffers."""
        L.dash_prefill_stage(self.p, k, self.Q, self.K, self.V, self.qbar, self.O, self.kbar, self.route,
                             self.workspace, stream=stream)

    def error_word(self) -> int:
        """Status word of the last call (0 = every bounded wait completed)."""
        off = L.dash_error_word_offset(self.p, L.DASH_OP_PREFILL)
        return int(self.workspace[off:off + 4].view(torch.int32).item())

    def __call__(self, stream=None):
        L.dash_prefill(self.p, self.Q, self.K, self.V, self.qbar, self.O, self.kbar, self.route, self.workspace,
                       stream=stream)
        return self.O

    def backward(self, dO, stream=None):
        """Gradients (fp32) of sum(dO * O) for the last call: dQ, dK, dV and dqbar [h_kv, d].  Needs
        want_route=True (the backward reads the forward's route lists and summaries)."""
        if self.route is None:
            raise ValueError("Prefill.backward needs the route lists: construct with want_route=True")
        assert dO.shape == self.O.shape and dO.dtype == self.O.dtype and dO.stride() == self.O.stride()
        if getattr(self, "_grads", None) is None:
            dev = self.Q.device
            ws = L.dash_workspace_size(self.p, L.DASH_OP_BACKWARD)
            self._bws = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)
            self._grads = (torch.empty(self.Q.shape, dtype=torch.float32, device=dev),
                           torch.empty(self.K.shape, dtype=torch.float32, device=dev),
                           torch.empty(self.V.shape, dtype=torch.float32, device=dev),
                           torch.empty((self.K.shape[2], self.Q.shape[3]), dtype=torch.float32, device=dev))
        dQ, dK, dV, dqbar = self._grads
        L.dash_backward(self.p, self.Q, self.K, self.V, self.qbar, dO, self.kbar, self.route, dQ, dK, dV, dqbar,
                        self._bws, stream=stream)
        return dQ, dK, dV, dqbar


def prefill(Q, K, V, qbar, **kw):
    return Prefill(Q, K, V, qbar, **kw)()


class DecodeState:
    """Caller-owned decode state: K/V caches, summary cache, incomplete-chunk state, lengths.

    Copying these tensors saves or restores a session."""

    def __init__(self, batch, capacity, h_q, h_kv, d, *, chunk, alpha, gamma, inv_sigma=1.0,
                 dtype=torch.bfloat16, device="cuda", qbar=None):
        self.K = torch.zeros((batch, capacity, h_kv, d), dtype=dtype, device=device)
        self.V = torch.zeros_like(self.K)
        self.T = capacity // chunk
        self.kbar = torch.zeros((batch, h_kv, self.T, d), dtype=torch.float32, device=device)
        self.state = torch.zeros((batch, h_kv, d + 2), dtype=torch.float32, device=device)
        self.seqlens = torch.zeros(batch, dtype=torch.int32, device=device)
        self.qbar = qbar
        self.O = torch.empty((batch, h_q, d), dtype=dtype, device=device)
        self.p = L.params(batch=batch, seqlen=capacity, h_q=h_q, h_kv=h_kv, d_h=d, chunk=chunk, alpha=alpha,
                          gamma=gamma, inv_sigma=inv_sigma, dtype=L.DASH_BF16 if dtype == torch.bfloat16 else L.DASH_F32,
                          k_strides=_st(self.K), v_strides=_st(self.V))
        ws = L.dash_workspace_size(self.p, L.DASH_OP_DECODE)
        self.workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=device)
        self.route = None

    def fill(self, K0, V0, lengths, stream=None):
        """Copy prefilled keys/values [b, L0, h_kv, d] in and build the summary cache (Eq. 4)."""
        L0 = K0.shape[1]
        self.K[:, :L0].copy_(K0)
        self.V[:, :L0].copy_(V0)
        self.seqlens.copy_(torch.as_tensor(lengths, dtype=torch.int32))
        L.dash_summary_build(self.p, self.K, self.qbar, self.seqlens, self.kbar, self.state, stream=stream)

    def append(self, k_new, v_new, stream=None):
        L.dash_summary_append(self.p, k_new, v_new, self.qbar, self.K, self.V, self.kbar, self.state,
                              self.seqlens, stream=stream)

    def decode(self, q, stream=None):
        L.dash_decode(self.p, q, self.K, self.V, self.kbar, self.seqlens, self.O, self.route, self.workspace,
                      stream=stream)
        return self.O

    def step(self, q, k_new, v_new, stream=None):
        self.append(k_new, v_new, stream)
        return self.decode(q, stream)

    def graph_step(self, q, k_new, v_new):
        """step() through a CUDA graph: the first call runs eagerly (one-time set-up stays out of
        the capture) and records append + decode on static input buffers; later calls copy the
        inputs in and replay.  The kernels read the lengths from device memory, so one graph
        serves every step."""
        if getattr(self, "_graph", None) is None:
            out = self.step(q, k_new, v_new)
            # one staging buffer holding q, k, v back to back (graph_step_packed fills it at once)
            self._stage = torch.empty(q.numel() + k_new.numel() + v_new.numel(), dtype=q.dtype, device=q.device)
            nq, nk = q.numel(), k_new.numel()
            self._qs = self._stage[:nq].view(q.shape)
            self._ks = self._stage[nq:nq + nk].view(k_new.shape)
            self._vs = self._stage[nq + nk:].view(v_new.shape)
            self._qs.copy_(q)
            self._ks.copy_(k_new)
            self._vs.copy_(v_new)
            self._graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self._graph):
                self.append(self._ks, self._vs)
                self.decode(self._qs)
            return out
        self._qs.copy_(q)
        self._ks.copy_(k_new)
        self._vs.copy_(v_new)
        self._graph.replay()
        return self.O

    @staticmethod
    def pack(q, k_new, v_new):
        """q, k, v of one step in the layout graph_step_packed takes (flattened, back to back)."""
        return torch.cat([q.reshape(-1), k_new.reshape(-1), v_new.reshape(-1)])

    def graph_step_packed(self, qkv):
        """graph_step with the step's q, k, v already packed (pack()): one copy in, then replay.
        The graph must exist (one graph_step call first)."""
        self._stage.copy_(qkv)
        self._graph.replay()
        return self.O

class PagedDecodeState:
    """DecodeState on paged K/V pools [num_pages, page_size, h_kv, d] with a page table
    [batch, max_pages] (device int32) that the caller may rewrite between steps; the summary
    cache and the incomplete-chunk state stay per sequence.  bf16, d = 128."""

    def __init__(self, batch, capacity, h_q, h_kv, d, *, chunk, alpha, gamma, page_size, num_pages,
                 page_table, inv_sigma=1.0, device="cuda", qbar=None):
        self.K = torch.zeros((num_pages, page_size, h_kv, d), dtype=torch.bfloat16, device=device)
        self.V = torch.zeros_like(self.K)
        self.page_table = page_table.to(device=device, dtype=torch.int32).contiguous()
        self.page_size = page_size
        self.T = capacity // chunk
        self.kbar = torch.zeros((batch, h_kv, self.T, d), dtype=torch.float32, device=device)
        self.state = torch.zeros((batch, h_kv, d + 2), dtype=torch.float32, device=device)
        self.seqlens = torch.zeros(batch, dtype=torch.int32, device=device)
        self.qbar = qbar
        self.O = torch.empty((batch, h_q, d), dtype=torch.bfloat16, device=device)
        row, head = h_kv * d, d
        self.p = L.params(batch=batch, seqlen=capacity, h_q=h_q, h_kv=h_kv, d_h=d, chunk=chunk, alpha=alpha,
                          gamma=gamma, inv_sigma=inv_sigma, dtype=L.DASH_BF16,
                          k_strides=(0, row, head), v_strides=(0, row, head))
        self.pk = L.paged_kv(self.page_table, page_size, num_pages, page_size * row, page_size * row)
        ws = L.dash_workspace_size(self.p, L.DASH_OP_DECODE)
        self.workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=device)
        self.route = None

    def fill(self, K0, V0, lengths, stream=None):
        """Copy the first lengths[b] prefilled keys/values of K0, V0 [b, L0, h_kv, d] into the
        sequences' pages and build the summary cache (Eq. 4)."""
        pt = self.page_table.cpu()
        for b in range(K0.shape[0]):
            n = int(lengths[b])
            for j in range((n + self.page_size - 1) // self.page_size):
                pid = int(pt[b, j])
                if not 0 <= pid < self.K.shape[0]:
                    raise ValueError(f"sequence {b}: page slot {j} holds prefilled tokens but is unmapped ({pid})")
                t0, t1 = j * self.page_size, min(n, (j + 1) * self.page_size)
                self.K[pid, :t1 - t0].copy_(K0[b, t0:t1])
                self.V[pid, :t1 - t0].copy_(V0[b, t0:t1])
        self.seqlens.copy_(torch.as_tensor(lengths, dtype=torch.int32))
        L.dash_summary_build_paged(self.p, self.pk, self.K, self.qbar, self.seqlens, self.kbar, self.state,
                                   stream=stream)

    def append(self, k_new, v_new, stream=None):
        L.dash_summary_append_paged(self.p, self.pk, k_new, v_new, self.qbar, self.K, self.V, self.kbar,
                                    self.state, self.seqlens, stream=stream)

    def decode(self, q, stream=None):
        L.dash_decode_paged(self.p, self.pk, q, self.K, self.V, self.kbar, self.seqlens, self.O, self.route,
                            self.workspace, stream=stream)
        return self.O

    def step(self, q, k_new, v_new, stream=None):
        self.append(k_new, v_new, stream)
        return self.decode(q, stream)
