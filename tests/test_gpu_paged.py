"""GPU parity of decoding on paged K/V caches (dash_summary_build_paged / dash_summary_append_paged /
dash_decode_paged through the C ABI).

Every paged step is checked against the float64 oracle directly (oracle.decode on the same
tokens: routed sets by the margin rule, outputs at the bf16 tolerance, the bitmask against the
lists) on a schedule of steps that includes the steps around a page move, and the paged summary
cache and incomplete-chunk state against oracle.stage0.  A paged pool holds the same tokens as a
contiguous cache, only scattered over pages in the order the page table gives, so in addition
every result must equal the contiguous calls bit for bit, step after step."""
import numpy as np
import pytest
import torch

import adaptive_sparse_hierarchical_b200 as D
from adaptive_sparse_hierarchical_b200 import inputs
from adaptive_sparse_hierarchical_b200.api import PagedDecodeState

from test_gpu_decode import _check_step, _check_summaries, _state

pytestmark = pytest.mark.gpu


def _table(rng, b, max_pages, num_pages, unmapped_from):
    """Distinct pool pages in random order; slots at or beyond unmapped_from[b] are -1."""
    ids = rng.permutation(num_pages)[:b * max_pages].reshape(b, max_pages).astype(np.int32)
    for bb in range(b):
        ids[bb, unmapped_from[bb]:] = -1
    return ids


@pytest.mark.parametrize("B,page_size", [(64, 128), (128, 128), (64, 256)])
def test_paged_decode_equals_contiguous(B, page_size):
    b, cap, hq, hkv, d = 3, 2048, 16, 2, 128
    steps = 150
    x = inputs.planted(31, b, cap, hq, hkv, d, B, dtype="bf16", chunk_frac=0.1)
    lengths = np.array([300, 1000, B])
    max_pages = cap // page_size
    num_pages = b * max_pages + 7
    rng = np.random.default_rng(5)
    # sequence 0 leaves its last slots unmapped: no kernel may touch them
    last = lengths + steps
    unmapped = [(int(last[0]) + page_size - 1) // page_size, max_pages, max_pages]
    table = torch.from_numpy(_table(rng, b, max_pages, num_pages, unmapped))

    qbar = torch.from_numpy(x["qbar"]).cuda()
    ref = _state(x, lengths, cap, chunk=B, alpha=1.5, gamma=6.0, dtype="bf16")
    pg = PagedDecodeState(b, cap, hq, hkv, d, chunk=B, alpha=1.5, gamma=6.0, page_size=page_size,
                          num_pages=num_pages, page_table=table, qbar=qbar)
    counts = torch.zeros_like(ref.rt[0])
    idx, bias, bm = torch.zeros_like(ref.rt[1]), torch.zeros_like(ref.rt[2]), torch.full_like(ref.bm, -1)
    pg.route = D.route_out(counts, idx, bias, bm)
    pg.rt, pg.bm = (counts, idx, bias), bm
    L0 = int(lengths.max())
    pg.fill(torch.from_numpy(x["K"][:, :L0]).to("cuda", torch.bfloat16),
            torch.from_numpy(x["V"][:, :L0]).to("cuda", torch.bfloat16), lengths)
    torch.cuda.synchronize()
    _check_summaries(pg, x, B)
    assert torch.equal(pg.kbar, ref.kbar)
    assert torch.equal(pg.state, ref.state)

    dev = {k: torch.from_numpy(x[k]).to("cuda", torch.bfloat16) for k in ("Q", "K", "V")}
    rows = torch.arange(b, device="cuda")
    for step in range(steps):
        pos = torch.from_numpy(lengths + step).long().cuda()
        q, k, v = (dev[n][rows, pos].contiguous() for n in ("Q", "K", "V"))
        o_ref = ref.step(q, k, v)
        o = pg.step(q, k, v)
        torch.cuda.synchronize()
        if step % 20 == 0 or step in (59, 61, 62):
            # the paged step against the float64 oracle on the same tokens
            L = lengths + step + 1
            _check_step(pg, x, x["Q"][np.arange(b), L - 1], L, chunk=B, alpha=1.5, gamma=6.0, dtype="bf16")
        assert torch.equal(o, o_ref), step
        assert torch.equal(pg.seqlens, ref.seqlens)
        if step == 60:
            # the caller moves one of sequence 1's pages to a free page between steps
            free = sorted(set(range(num_pages)) - set(table[table >= 0].tolist()))[0]
            old = int(table[1, 2])
            pg.K[free].copy_(pg.K[old])
            pg.V[free].copy_(pg.V[old])
            pg.K[old].zero_()
            pg.V[old].zero_()
            table[1, 2] = free
            pg.page_table.copy_(table)
    assert torch.equal(pg.kbar, ref.kbar)
    assert torch.equal(pg.state, ref.state)
    assert torch.equal(pg.rt[0], ref.rt[0]) and torch.equal(pg.bm, ref.bm)
    _check_step(pg, x, x["Q"][np.arange(b), last - 1], last, chunk=B, alpha=1.5, gamma=6.0, dtype="bf16")
    _check_summaries(pg, x, B)

    # the pool holds exactly the contiguous cache's tokens, at the places the table gives
    for bb in range(b):
        for j in range(int(last[bb])):
            pid = int(table[bb, j // page_size])
            if j % 97 == 0 or j == int(last[bb]) - 1:
                assert torch.equal(pg.K[pid, j % page_size], ref.K[bb, j]), (bb, j)
                assert torch.equal(pg.V[pid, j % page_size], ref.V[bb, j]), (bb, j)
