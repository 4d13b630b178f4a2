"""Pins of the oracle's attention (CPU only).

Definition pinned: xGR page ("xGR: Efficient Generative Recommendation Serving
at Scale"), 2.1 xAttention -- the Shared prompt KV, the beam's own Unshared
tokens, and the staged Shared / Unshared / Merging computation that yields the
plain softmax attention over all keys.  Each pin below would fail under a
plausible slip in the oracle: a missing scale or max shift, k/v swapped, a wrong
GQA head map, a dropped key group, a wrong ancestry index.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def rnd(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(torch.bfloat16)


def test_golden_two_keys(orc):
    fx = json.load(open(os.path.join(GOLDEN, "attention_tiny.json")))
    out, lse = orc.attend(bf(fx["q"]), bf(fx["k"]), bf(fx["v"]), scale=fx["scale"])
    env = {"exp": math.exp, "log": math.log}
    want = [eval(e, env) for e in fx["out_expr"]]
    assert np.allclose(out[0], want, rtol=0, atol=1e-15)
    assert abs(lse[0] - eval(fx["lse_expr"], env)) < 1e-15


def test_single_key_closed_form(orc):
    q, k, v = rnd((3, 64), 1), rnd((1, 64), 2), rnd((1, 64), 3)
    out, lse = orc.attend(q, k, v)
    qd, kd, vd = q.double().numpy(), k.double().numpy(), v.double().numpy()
    assert np.array_equal(out, np.repeat(vd, 3, axis=0))
    assert np.allclose(lse, (qd @ kd.T)[:, 0] / 8.0, atol=1e-13)


def test_identical_keys_closed_form(orc):
    N = 37
    q = rnd((2, 32), 4)
    k = rnd((1, 32), 5).repeat(N, 1)
    v = rnd((1, 32), 6).repeat(N, 1)
    out, lse = orc.attend(q, k, v)
    s0 = (q.double() @ k[:1].double().T).numpy()[:, 0] / math.sqrt(32)
    assert np.allclose(out, np.repeat(v[:1].double().numpy(), 2, axis=0), atol=1e-14)
    assert np.allclose(lse, s0 + math.log(N), atol=1e-12)


def test_zero_query_is_mean(orc):
    N = 50
    q = torch.zeros((1, 16), dtype=torch.bfloat16)
    k, v = rnd((N, 16), 7), rnd((N, 16), 8)
    out, lse = orc.attend(q, k, v)
    assert np.allclose(out[0], v.double().mean(0).numpy(), atol=1e-14)
    assert abs(lse[0] - math.log(N)) < 1e-13


def test_matches_library_sdpa(orc):
    """Library special case: torch's scaled_dot_product_attention in fp64."""
    q, k, v = rnd((9, 128), 10), rnd((300, 128), 11), rnd((300, 128), 12)
    out, lse = orc.attend(q, k, v)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double()[None], k.double()[None], v.double()[None])[0].numpy()
    s = (q.double() @ k.double().T) / math.sqrt(128)
    ref_lse = torch.logsumexp(s, dim=-1).numpy()
    assert np.allclose(out, ref, atol=1e-12)
    assert np.allclose(lse, ref_lse, atol=1e-12)


def _decode_case(seed, BW=4, Hq=8, Hkv=2, D=32, P=40, X=0, S=3, s=2, n_live=3):
    g = np.random.default_rng(seed)
    q = rnd((BW, Hq, D), seed + 1)
    ks, vs = rnd((Hkv, P, D), seed + 2), rnd((Hkv, P, D), seed + 3)
    kx, vx = (rnd((Hkv, X, D), seed + 4), rnd((Hkv, X, D), seed + 5)) if X else (None, None)
    kp, vp = rnd((S, BW, Hkv, D), seed + 6), rnd((S, BW, Hkv, D), seed + 7)
    anc = g.integers(0, BW, size=(BW, S)).astype(np.int32)
    anc[:, s] = np.arange(BW)
    return dict(q=q, ks=ks, vs=vs, kx=kx, vx=vx, kp=kp, vp=vp, anc=anc, s=s, n_live=n_live,
                BW=BW, Hq=Hq, Hkv=Hkv, D=D, P=P, X=X)


@pytest.mark.parametrize("X", [0, 11])
def test_decode_attention_gqa_matches_sdpa(orc, X):
    """Library special case over the explicitly concatenated keys, with GQA
    written the textbook way (kv heads repeated G times)."""
    c = _decode_case(20 + X, X=X)
    out, lse = orc.decode_attention(c["q"], c["ks"], c["vs"], c["kp"], c["vp"], c["anc"],
                                    c["s"], c["n_live"], c["kx"], c["vx"])
    G = c["Hq"] // c["Hkv"]
    for b in range(c["n_live"]):
        parts_k = [c["ks"]] + ([c["kx"]] if X else [])
        parts_v = [c["vs"]] + ([c["vx"]] if X else [])
        for i in range(c["s"] + 1):
            parts_k.append(c["kp"][i, c["anc"][b, i]][:, None, :])
            parts_v.append(c["vp"][i, c["anc"][b, i]][:, None, :])
        K = torch.cat(parts_k, dim=1).double().repeat_interleave(G, dim=0)   # [Hq][n][D]
        Vv = torch.cat(parts_v, dim=1).double().repeat_interleave(G, dim=0)
        Q = c["q"][b].double()[:, None, :]                                    # [Hq][1][D]
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, Vv)[:, 0].numpy()
        ref_lse = torch.logsumexp((Q @ K.transpose(1, 2))[:, 0] / math.sqrt(c["D"]), -1).numpy()
        assert np.allclose(out[b], ref, atol=1e-12)
        assert np.allclose(lse[b], ref_lse, atol=1e-12)


def test_dead_rows(orc):
    c = _decode_case(30, n_live=2)
    out, lse = orc.decode_attention(c["q"], c["ks"], c["vs"], c["kp"], c["vp"], c["anc"],
                                    c["s"], c["n_live"])
    assert np.all(out[2:] == 0) and np.all(np.isneginf(lse[2:]))
    assert np.all(np.isfinite(lse[:2]))


def test_bad_ancestry_slot_is_an_error(orc):
    c = _decode_case(31)
    c["anc"][1, 0] = c["BW"]
    with pytest.raises(RuntimeError):
        orc.decode_attention(c["q"], c["ks"], c["vs"], c["kp"], c["vp"], c["anc"], c["s"],
                             c["n_live"])


def _merge(parts):
    """Online-softmax merge of partial (O, LSE) pairs (the Merging stage)."""
    lses = np.stack([p[1] for p in parts])
    m = lses.max(0)
    w = np.exp(lses - m)
    lse = m + np.log(w.sum(0))
    out = sum(np.exp(p[1] - lse)[..., None] * p[0] for p in parts)
    return out, lse


def test_split_merge_equals_unsplit(orc):
    """The page's claim: Shared + Unshared stages merged by online softmax give
    the full attention.  Split the shared keys into random chunks as well."""
    c = _decode_case(40, P=90, X=13, s=2, n_live=4)
    out, lse = orc.decode_attention(c["q"], c["ks"], c["vs"], c["kp"], c["vp"], c["anc"],
                                    c["s"], c["n_live"], c["kx"], c["vx"])
    G, D = c["Hq"] // c["Hkv"], c["D"]
    rng = np.random.default_rng(41)
    cuts = sorted(rng.choice(np.arange(1, 90), size=3, replace=False))
    bounds = [0] + list(cuts) + [90]
    for b in range(c["n_live"]):
        for h in range(c["Hq"]):
            g = h // G
            qrow = c["q"][b, h][None]
            parts = []
            for lo, hi in zip(bounds[:-1], bounds[1:]):
                parts.append(orc.attend(qrow, c["ks"][g, lo:hi], c["vs"][g, lo:hi]))
            parts.append(orc.attend(qrow, c["kx"][g], c["vx"][g]))
            uk = torch.stack([c["kp"][i, c["anc"][b, i], g] for i in range(c["s"] + 1)])
            uv = torch.stack([c["vp"][i, c["anc"][b, i], g] for i in range(c["s"] + 1)])
            parts.append(orc.attend(qrow, uk, uv))
            mo, ml = _merge(parts)
            assert np.allclose(mo[0], out[b, h], atol=1e-12)
            assert abs(ml[0] - lse[b, h]) < 1e-12


def test_beam_subset_equals_full(orc):
    c = _decode_case(50, X=7, n_live=3)
    full, full_lse = orc.decode_attention(c["q"], c["ks"], c["vs"], c["kp"], c["vp"], c["anc"],
                                          c["s"], c["n_live"], c["kx"], c["vx"])
    ids = [2, 0, 3]
    sub, sub_lse = orc.decode_attention(c["q"][ids], c["ks"], c["vs"], c["kp"], c["vp"], c["anc"],
                                        c["s"], c["n_live"], c["kx"], c["vx"], beams=ids)
    assert np.array_equal(sub, full[ids]) and np.array_equal(sub_lse, full_lse[ids])
