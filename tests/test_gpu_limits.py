"""The largest batch the C ABI admits: M = 2^31 - 1 tokens with topk =
E_part = 1 (M * topk and M * E_part must stay below 2^31).  Layout only --
the row buffers of such a batch would not fit a GPU together -- checked in
closed form on the device, in chunks: token t is routed to expert t % 2, so
expert 0 holds the even tokens in order and expert 1 the odd ones, and with
one partition every token has exactly one dispatch row."""
import pytest
import torch

import combine_moe_layout_08_b200 as moe

pytestmark = pytest.mark.gpu
DEV = "cuda"
CHUNK = 1 << 28


@pytest.mark.parametrize("dedup", [False, True])
def test_layout_at_the_largest_batch(dedup):
    M = (1 << 31) - 1
    prob = moe.MoEProblem(M, 8, 2, 1, 1, dedup=dedup)
    n_even = (M + 1) // 2                        # experts 0 and 1: even and odd tokens
    idx = torch.empty((M, 1), dtype=torch.int32, device=DEV)
    flat = idx.view(-1)
    for t0 in range(0, M, CHUNK):
        t1 = min(M, t0 + CHUNK)
        flat[t0:t1] = torch.arange(t0, t1, dtype=torch.int64, device=DEV).remainder(2).int()
    po = torch.zeros(2, dtype=torch.int32, device=DEV)
    lay = moe.alloc_layout(prob, DEV)
    lay.status.fill_(-1)
    ws = torch.empty(moe.layout_workspace_size(prob), dtype=torch.uint8, device=DEV)
    moe.moe_layout(prob, idx, po, lay, ws)
    torch.cuda.synchronize()
    assert lay.status.item() == 0
    assert lay.expert_count.tolist() == [n_even, M - n_even]
    assert lay.expert_offset.tolist() == [0, n_even, M]
    assert lay.part_count.tolist() == [M] and lay.part_offset.tolist() == [0, M]
    for t0 in range(0, M, CHUNK):
        t1 = min(M, t0 + CHUNK)
        t = torch.arange(t0, t1, dtype=torch.int64, device=DEV)
        want_row = torch.where(t.remainder(2) == 0, t // 2, n_even + t // 2)
        assert torch.equal(lay.exp_row[t0:t1].long(), want_row), f"exp_row [{t0}, {t1})"
        # dispatch row r holds token: even tokens first, then odd ones
        r = t
        want_tok = torch.where(r < n_even, 2 * r, 2 * (r - n_even) + 1)
        if dedup:                                # one partition: dispatch row = token
            assert torch.equal(lay.disp_token[t0:t1].long(), t), f"disp_token [{t0}, {t1})"
            assert torch.equal(lay.disp_row[t0:t1].long(), t), f"disp_row [{t0}, {t1})"
            assert torch.equal(lay.exp_to_disp[t0:t1].long(), want_tok), f"exp_to_disp [{t0}, {t1})"
        else:
            assert torch.equal(lay.disp_token[t0:t1].long(), want_tok), f"disp_token [{t0}, {t1})"
    del idx, lay, ws
    torch.cuda.empty_cache()


# Tiles past the shared-memory id cache (16384 pairs), so ids are read from
# global memory: 148 tiles of 65504 tokens (topk = 1, every token on expert
# 0, so each tile counts 65504 for one expert), and one token more, which
# rounds the tiles up to 65536 tokens and leaves a short last tile.
# Closed form: exp_row = t.
@pytest.mark.parametrize("M", [148 * 65504, 148 * 65504 + 1])
@pytest.mark.parametrize("dedup", [False, True])
def test_layout_with_tiles_past_the_id_cache(M, dedup):
    prob = moe.MoEProblem(M, 8, 2, 1, 2, dedup=dedup)
    idx = torch.zeros((M, 1), dtype=torch.int32, device=DEV)
    po = torch.tensor([1, 0], dtype=torch.int32, device=DEV)
    lay = moe.alloc_layout(prob, DEV)
    lay.status.fill_(-1)
    ws = torch.empty(moe.layout_workspace_size(prob), dtype=torch.uint8, device=DEV)
    moe.moe_layout(prob, idx, po, lay, ws)
    torch.cuda.synchronize()
    assert lay.status.item() == 0
    assert lay.expert_count.tolist() == [M, 0]
    assert lay.expert_offset.tolist() == [0, 0, M]   # expert 1 (partition 0) first
    assert lay.part_count.tolist() == [0, M] and lay.part_offset.tolist() == [0, 0, M]
    t = torch.arange(M, dtype=torch.int32, device=DEV)
    assert torch.equal(lay.exp_row[:M], t)
    assert torch.equal(lay.disp_token[:M], t)
    if dedup:                                    # every token in partition 1 only
        dr = lay.disp_row[:2 * M].view(M, 2)
        assert bool((dr[:, 0] == -1).all()) and torch.equal(dr[:, 1], t)
        assert torch.equal(lay.exp_to_disp[:M], t)
    del idx, lay, ws
    torch.cuda.empty_cache()
