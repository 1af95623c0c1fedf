"""engram_table_grad_noalloc: the sparse table gradient for callers that cannot
allocate device memory (a host framework that owns every allocation, or a
runtime with a fixed memory pool).  It sorts in a
scratch array built into the library instead of a caller workspace, so its
results must equal those of engram_table_grad on the same inputs, bit for bit
(the reduction is deterministic), and equal the oracle's reduction.  Two
calls in a row check that the second does not depend on what the first left
in the shared array.

This file is collected last on purpose, so that a run stopping at its first
failure has run every other test before it."""
import numpy as np
import pytest
import torch

from hashed_gram_conditional_engram_b200 import engram as eg
from hashed_gram_conditional_engram_b200 import synth
from oracle import engram_oracle as O

pytestmark = pytest.mark.gpu

K, D_H = 8, 16
ROWS = synth.primes_at_most(5003, 2 * K)


def _cfg():
    return eg.make_cfg(K, D_H, 64, 1, 1000, 770, eg.F32, ROWS, np.ones((2 * K, 3), np.uint64))


def _inputs(seed, n_tok):
    rng = np.random.default_rng(seed)
    # Zipf-skewed slots: a few rows collect many tokens, most collect one
    idx = np.stack([np.minimum(rng.zipf(1.2, n_tok) - 1, P - 1) for P in ROWS], -1)
    idx = idx.astype(np.int32)
    de = rng.standard_normal((n_tok, 2 * K * D_H)).astype(np.float32)
    return torch.from_numpy(idx).cuda(), torch.from_numpy(de).cuda()


def _outputs(n_items):
    return (torch.empty(n_items, dtype=torch.int64, device="cuda"),
            torch.empty((n_items, D_H), dtype=torch.float32, device="cuda"),
            torch.zeros(1, dtype=torch.int32, device="cuda"))


def test_noalloc_equals_workspace_entry_point_on_two_calls_in_a_row():
    cfg = _cfg()
    J = 2 * K
    # the first call fills most of the built-in array, the second is smaller
    for seed, n_tok in ((11, eg.NOALLOC_MAX_ITEMS // J), (12, 1000)):
        idx, de = _inputs(seed, n_tok)
        k_ws, r_ws, u_ws = _outputs(n_tok * J)
        nb = eg.engram_workspace_size(cfg, eg.WS_TABLE_GRAD, n_tok)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        eg.engram_table_grad(cfg, idx, de, n_tok, k_ws, r_ws, u_ws, ws, nb)
        k_na, r_na, u_na = _outputs(n_tok * J)
        eg.engram_table_grad_noalloc(cfg, idx, de, n_tok, k_na, r_na, u_na)
        torch.cuda.synchronize()
        U = int(u_ws.item())
        assert U > 0 and int(u_na.item()) == U
        assert torch.equal(k_na[:U], k_ws[:U])
        assert torch.equal(r_na[:U].view(torch.int32), r_ws[:U].view(torch.int32))
    assert eg.engram_get_status() == 0


@pytest.mark.parametrize("n_tok", [1, 777, eg.NOALLOC_MAX_ITEMS // (2 * K)])
def test_noalloc_equals_oracle(n_tok):
    """Distinct rows ascending and each row's fp32 sum of its tokens' de
    segments in ascending token order, bit for bit against the oracle's
    deterministic reduction (one token; a ragged count; the array full)."""
    cfg = _cfg()
    idx, de = _inputs(100 + n_tok, n_tok)
    k, r, u = _outputs(n_tok * 2 * K)
    eg.engram_table_grad_noalloc(cfg, idx, de, n_tok, k, r, u)
    torch.cuda.synchronize()
    k_ref, r_ref = O.table_grad_segments_fast(idx.cpu().numpy(), de.cpu().numpy(), ROWS, D_H)
    U = int(u.item())
    assert U == len(k_ref)
    assert np.array_equal(k[:U].cpu().numpy(), k_ref)
    assert np.array_equal(r[:U].cpu().numpy().view(np.int32), r_ref.view(np.int32))
    assert eg.engram_get_status() == 0


def test_noalloc_rejects_inputs_beyond_its_array():
    cfg = _cfg()
    J = 2 * K
    n_tok = eg.NOALLOC_MAX_ITEMS // J + 1
    idx, de = _inputs(3, n_tok)
    k, r, u = _outputs(n_tok * J)
    with pytest.raises(eg.EngramError) as ex:
        eg.engram_table_grad_noalloc(cfg, idx, de, n_tok, k, r, u)
    assert ex.value.rc == -7
