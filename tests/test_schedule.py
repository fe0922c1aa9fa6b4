"""Host-side tests of the forward kernel's static schedule (attn_fwd_schedule,
no GPU): every work unit runs exactly once, the persistent CTAs get even
shares of the K/V blocks, and causal rounds stay on a few heads at a time so
that each head's K/V is read from device memory about once ("GPU 学习日报 Day
21", section 6: parallelism over query row blocks, causal blocks skipped)."""
import math

import pytest

import exact_attention_127_b200 as attn

SMS = 148


def blocks(pair, N, causal):
    """K/V blocks of a unit: the larger of its two Q tiles' block counts."""
    nkv = (N + 127) // 128
    n = 0
    for t in range(2):
        r0 = pair * 256 + t * 128
        if r0 < N:
            n = max(n, min(r0 // 128 + 1, nkv) if causal else nkv)
    return n


def loads(B, H, N, causal, grid, per_unit=2.0):
    """Per-CTA work in K/V blocks (+ a fixed cost per unit) under the schedule."""
    cta, slot = attn.fwd_schedule(B, H, N, causal, grid)
    P = (N + 255) // 256
    g = min(grid, B * H * P)
    load = [0.0] * g
    for u in range(B * H * P):
        load[int(cta[u])] += blocks(u % P, N, causal) + per_unit
    return load, cta, slot


SHAPES = [(1, 1, 1), (1, 1, 128), (1, 1, 129), (1, 2, 300), (2, 3, 1000), (4, 16, 8192),
          (1, 16, 32768), (2, 16, 8192), (3, 16, 8192), (8, 16, 2048), (32, 32, 512),
          (1, 1, 8192), (5, 7, 2900), (1, 3, 768), (2, 5, 1280)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,N", SHAPES)
@pytest.mark.parametrize("grid", [1, 7, SMS])
def test_every_unit_once(B, H, N, causal, grid):
    cta, slot = attn.fwd_schedule(B, H, N, causal, grid)
    n_units = B * H * ((N + 255) // 256)
    g = min(grid, n_units)
    assert int(cta.min()) >= 0 and int(cta.max()) < g
    pairs = {(int(c), int(s)) for c, s in zip(cta.tolist(), slot.tolist())}
    assert len(pairs) == n_units                       # no two units share a CTA slot
    per_cta = [0] * g
    for c in cta.tolist():
        per_cta[c] += 1
    for c in range(g):                                 # slots of a CTA are 0 .. count-1
        got = sorted(int(s) for cc, s in zip(cta.tolist(), slot.tolist()) if cc == c)
        assert got == list(range(per_cta[c]))


@pytest.mark.parametrize("B,H,N,floor", [(4, 16, 8192, 0.99), (1, 16, 32768, 0.99),
                                         (8, 16, 4096, 0.98), (1, 32, 16384, 0.99),
                                         (2, 16, 8192, 0.94)])
def test_causal_balance(B, H, N, floor):
    load, _, _ = loads(B, H, N, True, SMS)
    assert sum(load) / len(load) / max(load) >= floor


def test_noncausal_balance():
    for (B, H, N) in ((8, 16, 2048), (32, 32, 512)):
        load, _, _ = loads(B, H, N, False, SMS)
        assert max(load) - min(load) <= blocks(0, N, False) + 2.0


def test_causal_rounds_stay_on_few_heads():
    """Headline shape: in each of the first rounds every CTA runs one mirror job
    (units P-1-m and m of one head, 2P+2 blocks together), and the jobs of a round
    cover only ceil(148 / 16) + 1 consecutive heads."""
    B, H, N = 4, 16, 8192
    P = N // 256
    cta, slot = attn.fwd_schedule(B, H, N, True, SMS)
    by = {}
    for u in range(B * H * P):
        by[(int(cta[u]), int(slot[u]))] = (u // P, u % P)
    jobs_per_round = SMS
    for r in range(3):
        heads = set()
        for c in range(SMS):
            bh0, p0 = by[(c, 2 * r)]
            bh1, p1 = by[(c, 2 * r + 1)]
            assert bh0 == bh1 and p0 + p1 == P - 1 and p0 > p1
            heads.add(bh0)
        assert max(heads) - min(heads) + 1 <= math.ceil(jobs_per_round / (P // 2)) + 1


def test_causal_tail_longest_first():
    """After the mirror rounds, a CTA's units never grow longer."""
    B, H, N = 4, 16, 8192
    P = N // 256
    cta, slot = attn.fwd_schedule(B, H, N, True, SMS)
    seq = {}
    for u in range(B * H * P):
        seq.setdefault(int(cta[u]), []).append((int(slot[u]), u % P))
    for c, lst in seq.items():
        lst.sort()
        tail = [p for s, p in lst if s >= 2 * 5]      # 5 mirror rounds at this shape
        assert tail == sorted(tail, reverse=True)


def test_rejects_bad_arguments():
    with pytest.raises(attn.AttnError):
        attn.fwd_schedule(1, 1, 128, True, 0)
    with pytest.raises(attn.AttnError):
        attn.fwd_schedule(-1, 1, 128, True, 4)
