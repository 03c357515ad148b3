"""The seeded input generators (workloads.py) produce the recipe they state:
byte-identical per seed, the outlier channels, the mixture-of-experts
routing (top-k distinct experts per token, segments padded to 128 rows with
zero rows), and the long packed batch (sequences padded to 128).  CPU only."""
import numpy as np
import torch

import workloads as wl


def test_same_seed_same_bytes():
    a = wl.normal_bf16((64, 256), 0.02, 5)
    b = wl.normal_bf16((64, 256), 0.02, 5)
    c = wl.normal_bf16((64, 256), 0.02, 6)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert not torch.equal(a.view(torch.int16), c.view(torch.int16))
    X1, W1, d1 = wl.llama_layer("o_proj", seed=1, M=128)
    X2, W2, d2 = wl.llama_layer("o_proj", seed=1, M=128)
    assert all(torch.equal(p.view(torch.int16), q.view(torch.int16))
               for p, q in [(X1, X2), (W1, W2), (d1, d2)])


def test_outlier_channels():
    K = 4096
    x = wl.activations_with_outliers(512, K, 3).float()
    rms = x.pow(2).mean(0).sqrt()
    big = torch.nonzero(rms > 10).flatten()
    assert len(big) == round(0.001 * K)                     # 4 channels x50
    assert float(rms[big].min()) > 40 and float(rms[rms <= 10].max()) < 1.3


def test_moe_routing_structure():
    r = wl.moe_routing(0)
    G, T, k = wl.MOE_EXPERTS, wl.MOE_TOKENS, wl.MOE_TOPK
    off = np.array(r.offsets)
    assert len(off) == G + 1 and off[0] == 0 and np.all(off % 128 == 0) and np.all(np.diff(off) >= 0)
    assert sum(r.counts) == T * k and r.m_total_pad == off[-1]
    assert np.all(np.diff(off) == (np.array(r.counts) + 127) // 128 * 128)
    rt = r.row_token.numpy()
    assert (rt == -1).sum() == r.m_total_pad - T * k
    # every token routed to exactly k distinct experts
    seen = np.zeros(T, np.int64)
    for e in range(G):
        seg = rt[off[e]:off[e] + r.counts[e]]
        assert np.all(seg >= 0) and np.all(np.diff(seg) > 0)       # stable by token, distinct
        assert np.all(rt[off[e] + r.counts[e]:off[e + 1]] == -1)  # padding after the rows
        seen[seg] += 1
    assert np.all(seen == k)
    # Zipf(1.1) popularity: the busiest expert sees far more tokens than the median one
    c = np.sort(np.array(r.counts))
    assert c[-1] > 4 * c[G // 2]


def test_moe_permuted_rows():
    r = wl.moe_routing(0)
    width = 256
    P = wl.moe_permuted(r, width, 1.0, 11)
    base = wl.normal_bf16((wl.MOE_TOKENS, width), 1.0, 11)
    rt = r.row_token
    valid = rt >= 0
    assert torch.equal(P[valid].view(torch.int16), base[rt[valid]].view(torch.int16))
    assert torch.all(P[~valid] == 0)


def test_packed_batch_padding():
    mask = wl.packed_rows_mask(0)
    lens = wl.packed_lengths(0)
    assert len(mask) == wl.PACKED_TOKENS and all(1024 <= L <= 16384 for L in lens)
    pos = 0
    for L in lens:
        if pos >= wl.PACKED_TOKENS:
            break
        n = min(L, wl.PACKED_TOKENS - pos)
        assert bool(mask[pos:pos + n].all())
        pad_end = min(pos + (L + 127) // 128 * 128, wl.PACKED_TOKENS)
        assert not bool(mask[pos + n:pad_end].any())
        pos += (L + 127) // 128 * 128
    x = wl.packed_activations(256, 0, total=wl.PACKED_TOKENS)
    assert torch.all(x[~mask] == 0)
    # Student-t with nu = 3: heavy tails (excess kurtosis far above a normal's 0)
    v = x[mask].float().flatten()
    kurt = float(((v - v.mean()) ** 4).mean() / v.var() ** 2) - 3.0
    assert kurt > 3.0


def test_packed_segments_match_mask():
    """The segment table of the packing marks exactly the mask's real tokens,
    with 128-aligned segment starts covering the whole batch."""
    off, ln = wl.packed_segments(0)
    mask = wl.packed_rows_mask(0)
    assert off[0] == 0 and off[-1] == wl.PACKED_TOKENS
    assert all(o % 128 == 0 for o in off)
    want = torch.zeros(wl.PACKED_TOKENS, dtype=torch.bool)
    for a, n in zip(off, ln):
        want[a:a + n] = True
    assert torch.equal(want, mask)
