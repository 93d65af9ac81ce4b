"""Host-side check of the fused decode kernel's attention schedule (no GPU).

The kernel splits the 64-key chunks of every (batch row, head) pair evenly
over its CTAs.  Each CTA holds a fixed number of pair slots, and the next
stage's gather reads a fixed number of contributing CTAs per pair.  Both
limits must hold for ANY mix of lengths the host accepts, because the
lengths only exist on the device.  The schedule is restated here from its
definition: pairs get max(nk_b, m) entries on the first Ga CTAs.  The
bounds are checked over random and adversarial length mixes, together
with the bookkeeping the kernel relies on:
  * each pair's contributor list covers exactly the CTAs that write its
    partials;
  * exactly one CTA appends each pair's new key and value;
  * every real chunk is streamed once;
  * equal lengths are never padded.
The per-CTA limits are read from the kernel source, so the test follows
the kernel's constants.
"""
import os
import random
import re

import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "rank_transformer_b200", "csrc", "decode_fused.cu")


def _const(name):
    m = re.search(r"constexpr int %s = (\d+);" % name, open(SRC).read())
    assert m, name
    return int(m.group(1))


CMAX, MAXP, MAXSU = _const("DF_CMAX"), _const("DF_MAX_PAIRS"), _const("DF_MAX_SU")


def accepted(B, H, G, S_max):
    """The host's acceptance rule for the attention schedule."""
    Ga = min(G, (CMAX - 1) * H)
    return (MAXP - 1) * Ga >= 2 * B * H and B * H * ((S_max + 63) // 64) * Ga < 2 ** 31


def schedule(pos, H, G, S_max):
    B = len(pos)
    L = [min(max(p, 0), S_max - 1) + 1 for p in pos]
    nk = [(l + 63) // 64 for l in L]
    raw = H * sum(nk)
    Ga = min(G, (CMAX - 1) * H)
    den = (MAXP - 1) * Ga - B * H
    m = max(1, -(-raw // den)) if den > 0 else 1
    ne = [max(k, m) for k in nk]
    pre = [0]
    for b in range(B):
        pre.append(pre[-1] + H * ne[b])
    return dict(L=L, nk=nk, ne=ne, pre=pre, Ga=Ga, m=m, C=pre[-1])


def entry(s, c):
    b = 0
    while b + 1 < len(s["pre"]) - 1 and c >= s["pre"][b + 1]:
        b += 1
    r = c - s["pre"][b]
    return b, r // s["ne"][b], r % s["ne"][b]


def share(s, g):
    if g >= s["Ga"]:
        return 0, 0
    return g * s["C"] // s["Ga"], (g + 1) * s["C"] // s["Ga"]


def owner(c, C, G):
    return ((c + 1) * G - 1) // C


def check(pos, H, G, S_max):
    s = schedule(pos, H, G, S_max)
    B, C, Ga = len(pos), s["C"], s["Ga"]
    writers, appends, streamed = {}, {}, 0
    for g in range(G):
        c0, c1 = share(s, g)
        if c0 >= c1:
            continue
        b0, h0, _ = entry(s, c0)
        b1, h1, _ = entry(s, c1 - 1)
        pf, npairs = b0 * H + h0, b1 * H + h1 - (b0 * H + h0) + 1
        assert npairs <= MAXP, (pos, H, G, g, npairs)
        su = 0
        for c in range(c0, c1):
            b, h, kc = entry(s, c)
            streamed += kc < s["nk"][b]
            if c == c1 - 1 or c == s["pre"][b] + h * s["ne"][b] + s["ne"][b] - 1:
                writers.setdefault((b, h), []).append((g, su))
                su += 1
        assert su <= MAXSU
        for pair in range(pf, pf + npairs):
            b, h = divmod(pair, H)
            if owner(s["pre"][b] + h * s["ne"][b] + s["nk"][b] - 1, C, Ga) == g:
                appends[(b, h)] = appends.get((b, h), 0) + 1
    assert streamed == H * sum(s["nk"])
    for b in range(B):
        for h in range(H):
            e0 = s["pre"][b] + h * s["ne"][b]
            slots = []
            for gg in range(owner(e0, C, Ga), owner(e0 + s["ne"][b] - 1, C, Ga) + 1):
                if C < Ga and (gg + 1) * C // Ga == gg * C // Ga:
                    continue
                b2, h2, _ = entry(s, gg * C // Ga)
                su = b * H + h - (b2 * H + h2)
                assert 0 <= su < MAXSU and len(slots) < CMAX, (pos, H, G, b, h)
                slots.append((gg, su))
            assert sorted(slots) == sorted(writers[(b, h)]), (pos, H, b, h)
            assert appends.get((b, h)) == 1, (pos, H, b, h)
    if len(set(pos)) == 1:
        assert s["ne"] == s["nk"], (pos, H)
    return s


@pytest.mark.parametrize("G", [132, 148])
@pytest.mark.parametrize("H", [1, 2, 4, 8, 12, 32, 40, 64, 128])
def test_attention_schedule_limits_hold_for_any_lengths(G, H):
    rng = random.Random(1000 * G + H)
    S_max = 16384
    for B in (1, 2, 3, 4):
        if not accepted(B, H, G, S_max):
            continue
        cases = [[S_max - 1] * B, [0] * B, [S_max - 1] + [0] * (B - 1),
                 [0] * (B - 1) + [S_max - 1], [63, 64, 65, 127][:B]]
        cases += [[rng.randint(0, S_max - 1) for _ in range(B)] for _ in range(12)]
        cases += [[rng.choice([0, 1, 62, 63, 64, 4095, S_max - 1]) for _ in range(B)]
                  for _ in range(12)]
        for pos in cases:
            check(pos, H, G, S_max)


def test_skewed_batch_is_padded_and_equal_batch_is_not():
    s = schedule([16319, 4095, 1023, 63], 32, 148, 16384)
    assert s["m"] > 1 and s["ne"][3] == s["m"] > s["nk"][3]
    s = schedule([2047] * 4, 32, 148, 2176)
    assert s["ne"] == s["nk"]


def test_few_heads_use_fewer_ctas():
    # 4 heads: a pair may span at most CMAX CTAs, so attention runs on 14 * 4
    s = check([3999], 4, 148, 4000)
    assert s["Ga"] == (CMAX - 1) * 4 < 148
