"""The stream-K partition of the few-token GEMM, checked on the CPU.

The kernel deals the W x KT (weight tile, k-tile) iterations to G CTAs in
contiguous shares [c T / G, (c+1) T / G) and finds the CTA that owns
iteration i as ((i + 1) G - 1) // T; the host shrinks G from
min(SMs, T, 8 W) until no tile has more than 9 contributing CTAs (one slab
slot each), and splits nothing when whole tiles already occupy more than
3/4 of the SMs. These mirror the formulas in csrc/gemm_skinny.cuh (cta_of,
SegIter) and csrc/nvfp4_api.cu (skinny_stream_k_grid) and check the
properties the kernel depends on, over a sweep of shapes.
"""
import pytest

MAX_SPLITS, MAX_CONTRIB = 8, 9


def owner(i, T, G):
    return ((i + 1) * G - 1) // T


def grid(sms, W, KT):
    if 4 * W > 3 * sms:
        return 0
    T = W * KT
    G = min(sms, T, W * MAX_SPLITS)
    while G > W:
        worst = max(owner((w + 1) * KT - 1, T, G) - owner(w * KT, T, G) + 1 for w in range(W))
        if worst <= MAX_CONTRIB:
            return G
        G -= 1
    return 0


def segments(c, W, KT, G):
    T = W * KT
    i, i1 = c * T // G, (c + 1) * T // G
    out = []
    while i < i1:
        wt, k0 = divmod(i, KT)
        k1 = min(KT, k0 + (i1 - i))
        out.append((wt, k0, k1))
        i += k1 - k0
    return out


@pytest.mark.parametrize("sms", [148, 132, 20])
@pytest.mark.parametrize("W,KT", [(1, 1), (1, 68), (8, 8), (40, 68), (136, 20), (147, 3),
                                  (3, 5), (12, 17), (100, 1)])
def test_stream_k_partition(sms, W, KT):
    G = grid(sms, W, KT)
    if 4 * W > 3 * sms:
        assert G == 0
        return
    assert W < G <= min(sms, W * KT, W * MAX_SPLITS) or G == 0
    if G == 0:
        return
    T = W * KT
    covered = []
    contrib = {w: [] for w in range(W)}
    for c in range(G):
        segs = segments(c, W, KT, G)
        assert segs, "every CTA has work"
        assert len(segs) <= 2, "a share is shorter than a tile, so it spans at most two"
        for wt, k0, k1 in segs:
            assert 0 <= k0 < k1 <= KT
            covered.extend(wt * KT + k for k in range(k0, k1))
            contrib[wt].append(c)
            for k in range(k0, k1):
                assert owner(wt * KT + k, T, G) == c
    assert covered == list(range(T)), "shares tile the iterations exactly, in order"
    for w, cs in contrib.items():
        assert cs == list(range(owner(w * KT, T, G), owner((w + 1) * KT - 1, T, G) + 1))
        assert len(cs) <= MAX_CONTRIB
