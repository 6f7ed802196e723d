"""The attention tile schedule: every (sequence, query-tile pair, head) item appears exactly once,
in batches of a few (sequence, head) groups, heaviest pair first inside a batch.

The schedule is the first part of the attention step's workspace: a header (item count), the
sequences' (start, length), then one packed entry per item (sequence | pair << 32 | head << 48).
"""
import numpy as np
import pytest
import torch

from tests.gpu_util import dev


@pytest.fixture(scope="module")
def hstu():
    import hstu_sequential_transduction_layer_b200 as m
    return m


@pytest.mark.gpu
@pytest.mark.parametrize("lengths,hd,H", [([300, 1, 129, 513, 0, 2000, 256, 257], 64, 2),
                                          ([4096, 4096, 100, 3000, 700], 128, 2),
                                          ([700] * 40 + [1] * 9 + [5000], 64, 2),
                                          # K/V above 256 MB: dynamic claiming, batches of 8 groups
                                          ([8192] * 7 + [4000, 2500, 700, 100, 1, 4096], 128, 8)])
def test_schedule_is_a_batched_heaviest_first_permutation(hstu, lengths, hd, H):
    d = H * hd
    lengths = np.asarray(lengths, dtype=np.int64)
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T = int(offsets[-1])
    uvqk = torch.zeros((T, 4 * d), dtype=torch.bfloat16, device="cuda")
    max_len = int(lengths.max())
    s = hstu.make_shape(len(lengths), T, max_len, d, H, hd, hd, hstu.HSTU_BF16, 32, 8)
    ws = torch.zeros(hstu.attention_workspace_size(s), dtype=torch.uint8, device="cuda")
    av = torch.empty((T, H * hd), dtype=torch.float32, device="cuda")
    hstu.hstu_attention_fwd(s, uvqk, dev(offsets), None, None, None, None, 1.0, av, ws)
    assert hstu.device_status() == hstu.HSTU_OK
    raw = ws.cpu().numpy().view(np.int64)
    B = len(lengths)
    n_items = int(raw[0])
    seqinfo_words = ((16 * B + 255) // 256) * 256 // 8
    items = raw[32 + seqinfo_words: 32 + seqinfo_words + n_items]
    seq, pair, head = items & 0xFFFFFFFF, (items >> 32) & 0xFFFF, items >> 48
    pairs = (lengths + 255) // 256
    expected = sorted((s_, m, h) for s_ in range(B) for h in range(H) for m in range(pairs[s_]))
    got = sorted(zip(seq.tolist(), pair.tolist(), head.tolist()))
    assert got == expected                                # each item exactly once
    # batches of gb (sequence, head) groups, sequences ranked by decreasing pair count; inside a
    # batch the pair index never increases and the batch starts with its heaviest item
    kv_per_group = 4 * hd * (((max_len + 255) // 256) * 256)
    dynamic = 4 * hd * T * H > (256 << 20)
    gb = max(1, min(256, (32 << 20) // kv_per_group)) if dynamic else 1 << 30
    rank_pairs = sorted(pairs[pairs > 0], reverse=True)
    group_pairs = np.repeat(rank_pairs, H)
    pos = 0
    for b0 in range(0, len(group_pairs), gb):
        cnt = int(group_pairs[b0:b0 + gb].sum())
        batch_pairs = pair[pos:pos + cnt]
        assert np.all(np.diff(batch_pairs) <= 0), "pairs must not increase inside a batch"
        assert int(batch_pairs[0]) == int(group_pairs[b0]) - 1   # heaviest item first
        pos += cnt
    assert pos == n_items


@pytest.mark.gpu
@pytest.mark.parametrize("lengths,hd,H", [([300, 1, 129, 513, 0, 2000, 256, 257], 64, 2),
                                          ([700] * 40 + [1] * 9 + [5000], 64, 3),
                                          ([8192] * 3 + [4000, 2500, 700, 100, 1], 64, 8),
                                          ([4096, 4096, 100, 3000, 700], 128, 4)])
def test_backward_schedule_is_a_heaviest_first_permutation(hstu, lengths, hd, H):
    """The attention backward's schedule (items: sequence | key tile << 32 | head << 48): every
    (sequence, key tile, head) item exactly once, by non-increasing cost (the query tiles the item
    visits, tiles - key tile), which the query-stationary dQ kernel at head dim 128 reads as the
    key tiles of query tile tiles - 1 - key tile."""
    d = H * hd
    lengths = np.asarray(lengths, dtype=np.int64)
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T = int(offsets[-1])
    B = len(lengths)
    uvqk = torch.zeros((T, 4 * d), dtype=torch.bfloat16, device="cuda")
    dav = torch.zeros((T, d), dtype=torch.bfloat16, device="cuda")
    max_len = int(lengths.max())
    s = hstu.make_shape(B, T, max_len, d, H, hd, hd, hstu.HSTU_BF16, 0, 0)
    ws = torch.zeros(int(hstu.library().hstu_attention_bwd_workspace_size(s)), dtype=torch.uint8,
                     device="cuda")
    f = lambda: torch.empty((T, d), dtype=torch.float32, device="cuda")
    hstu.hstu_attention_bwd(s, uvqk, dev(offsets), None, None, None, None, 1.0, dav, f(), f(), f(),
                            None, None, ws)
    torch.cuda.synchronize()
    assert hstu.device_status() == hstu.HSTU_OK
    raw = ws.cpu().numpy().view(np.int64)
    n_items = int(raw[0])
    seqinfo_words = ((16 * B + 255) // 256) * 256 // 8
    items = raw[32 + seqinfo_words: 32 + seqinfo_words + n_items]
    seq, jt, head = items & 0xFFFFFFFF, (items >> 32) & 0xFFFF, items >> 48
    tiles = (lengths + 127) // 128
    expected = sorted((s_, j, h) for s_ in range(B) for h in range(H) for j in range(tiles[s_]))
    got = sorted(zip(seq.tolist(), jt.tolist(), head.tolist()))
    assert got == expected                                # each item exactly once
    cost = tiles[seq] - jt
    assert np.all(np.diff(cost) <= 0), "heaviest first"
    assert int(cost[0]) == int(tiles.max())
