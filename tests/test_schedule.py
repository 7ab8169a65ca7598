"""The persistent attention schedule, checked on the CPU: the library's own host planner
(through the qattn_debug_attention_plan hook) combined with the rules the kernels follow for
dense launches (the attention kernel's segment list per CTA, the combine kernel's search for the
parts of a cut pair), written out below from their documented definitions.  For many shapes and
SM counts: every key step of every pair of Q tiles runs exactly once, partial-result slots are
unique and fit the workspace, the combine finds exactly the parts of each cut pair, and the key
steps per CTA are balanced to within one tail range."""
import numpy as np
import pytest

from precision_quantized_attention_b200 import _lib

NQ, BLOCK_M = 2, 128            # Q tiles per pair, rows per tile


def segments(p, c):
    """(pair, kv0, kv1, slot) of CTA c, in order: its whole pairs c, c + G, ..., then at most two
    tail segments from key steps [c * tail_w, (c + 1) * tail_w) of the tail pairs laid end to
    end; a segment covering only part of a pair writes partial slot 2c (first) or 2c + 1."""
    out = [(c + i * p["ctas"], 0, p["nkv"], -1) for i in range(p["whole"])]
    nkv, w = p["nkv"], p["tail_w"]
    end = p["tail_pairs"] * nkv
    for k in (0, 1):
        g0 = c * w
        g1 = min(g0 + w, end)
        if k == 1:
            g0 = (g0 // nkv + 1) * nkv          # the second segment starts at a pair start
        if g0 >= g1:
            break
        tp = g0 // nkv
        kv0 = g0 - tp * nkv
        kv1 = min(nkv, kv0 + (g1 - g0))
        slot = -1 if (kv0 == 0 and kv1 == nkv) else 2 * c + k
        out.append((p["whole"] * p["ctas"] + tp, kv0, kv1, slot))
    return out


def combine_parts(p, tp):
    """(CTA, slot) pairs the combine kernel merges for tail pair tp; empty when one CTA ran the
    whole pair."""
    w, nkv = p["tail_w"], p["nkv"]
    g0 = tp * nkv
    c_first, c_last = g0 // w, (g0 + nkv - 1) // w
    if c_first == c_last:
        return set()
    return {(c, 2 * c + (1 if c * w < g0 else 0)) for c in range(c_first, c_last + 1)}


SHAPES = [(1, 24, 8704, 128), (1, 24, 4608, 128), (1, 2, 256, 64), (2, 3, 777, 64),
          (1, 160, 1024, 64), (1, 2, 1000, 128), (1, 1, 1, 128), (4, 24, 8704, 128),
          (1, 24, 300, 64), (3, 7, 5000, 128)]


@pytest.mark.parametrize("num_sms", [148, 132, 64, 7, 2, 1, 200])
@pytest.mark.parametrize("B,H,L,D", SHAPES)
def test_every_key_step_once_and_parts_found(B, H, L, D, num_sms):
    p = _lib.debug_attention_plan(B, H, L, D, num_sms)
    pairs = p["pairs_per_head"] * H * B
    nkv = p["nkv"]
    assert p["pairs_per_head"] == -(-L // (NQ * BLOCK_M)) and nkv == -(-L // 128)
    assert 1 <= p["ctas"] <= num_sms
    assert 1 <= p["tail_w"] <= nkv

    runs = np.zeros((pairs, nkv), dtype=np.int32)
    slots, per_cta, parts_of = set(), [], {}
    for c in range(p["ctas"]):
        steps = 0
        for pair, kv0, kv1, slot in segments(p, c):
            assert 0 <= pair < pairs and 0 <= kv0 < kv1 <= nkv
            runs[pair, kv0:kv1] += 1
            steps += kv1 - kv0
            if slot >= 0:
                assert slot not in slots and slot < 2 * p["ctas"]
                slots.add(slot)
                parts_of.setdefault(pair, set()).add((c, slot))
        per_cta.append(steps)
    assert (runs == 1).all(), "a key step ran twice or never"

    # workspace: partial O rows and (max, sum) per slot, only when some pair is cut
    need = 2 * p["ctas"] * NQ * BLOCK_M * (D + 2) * 4
    assert p["workspace_bytes"] == (need if slots else 0)
    assert bool(slots) == (p["tail_w"] < nkv)

    # the combine kernel finds exactly the parts that were written
    for tp in range(p["tail_pairs"]):
        pair = p["whole"] * p["ctas"] + tp
        assert combine_parts(p, tp) == parts_of.get(pair, set())

    # balance: every CTA runs its whole pairs plus at most one tail range
    assert max(per_cta) <= p["whole"] * nkv + p["tail_w"]
    assert max(per_cta) - min(per_cta) <= p["tail_w"]


def test_documented_schedules():
    # L=8704, H=24 on 148 SMs: 816 pairs = 5 whole per CTA + 76 tail pairs cut into 35-step ranges
    p = _lib.debug_attention_plan(1, 24, 8704, 128, 148)
    assert (p["ctas"], p["whole"], p["tail_pairs"], p["nkv"], p["tail_w"]) == (148, 5, 76, 68, 35)
    # L=4608: the even share would be 34 of 36 steps (>= 0.8 of a pair): tail pairs stay whole
    p = _lib.debug_attention_plan(1, 24, 4608, 128, 148)
    assert p["tail_w"] == p["nkv"] == 36 and p["workspace_bytes"] == 0
    # fewer pairs than SMs: one CTA per pair, nothing cut
    p = _lib.debug_attention_plan(1, 2, 256, 64, 148)
    assert (p["ctas"], p["whole"], p["tail_pairs"]) == (2, 1, 0)


def test_plan_rejects_what_the_forward_rejects():
    for args in ((0, 1, 128, 128, 148), (1, 1, 128, 96, 148), (1, 1, 0, 128, 148),
                 (1, 1, 128, 128, 0)):
        with pytest.raises(_lib.QattnError):
            _lib.debug_attention_plan(*args)
