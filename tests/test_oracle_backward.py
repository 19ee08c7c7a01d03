"""Pins for the fp64 backward oracle (oracle_attend_backward).

The gate is a hard top-k choice through which no gradient flows (wispaper.ai
blog, "The Change"), so the backward is the gradient of softmax attention
over each row's fixed key set.  The C oracle writes that gradient out term
by term; these tests tie it to computations that share none of its code:
  * torch autograd through fp64 masked scaled-dot-product attention over the
    same token mask (the brute-force mask of oracle/bruteforce.py);
  * central finite differences of that forward on sampled entries;
  * identities that hold exactly: sum over keys of dV equals the sum of dO
    over the rows and heads of the group (each row's probabilities sum to
    one), and the sum over keys of dK is zero (each row's dS sums to zero);
  * dQ does not change when every key is shifted by the same vector.
Inputs are tiny (a few dozen tokens) so every row is checked.
"""
import numpy as np
import pytest
import torch

from oracle import Oracle, bruteforce as bf

SCALE_D = 8


def _bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(
        torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _problem(seed, lengths=(28, 20), Hq=4, Hkv=2, d=SCALE_D, B=8, k=3, integer=False):
    rng = np.random.default_rng(seed)
    T = sum(lengths)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    if integer:
        q = rng.integers(-3, 4, size=(T, Hq, d)).astype(np.float32)
        kk = rng.integers(-3, 4, size=(T, Hkv, d)).astype(np.float32)
    else:
        q = rng.standard_normal((T, Hq, d)).astype(np.float32)
        kk = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    v = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    dO = rng.standard_normal((T, Hq, d)).astype(np.float32)
    return dict(cu=cu, q=_bits(q), k=_bits(kk), v=_bits(v), dO=_bits(dO), Hq=Hq, Hkv=Hkv,
                d=d, B=B, k_top=k, T=T)


def _oracle(P, kbits=None):
    return Oracle(P["q"], P["k"] if kbits is None else kbits, P["v"], P["cu"], P["Hq"],
                  P["Hkv"], P["d"], P["B"], P["k_top"])


def _all_rows(P):
    return np.arange(P["T"], dtype=np.int64)


def _torch_grads(P, sel):
    """dQ, dK, dV by autograd of fp64 masked SDPA, head by head."""
    T, Hq, Hkv, d = P["T"], P["Hq"], P["Hkv"], P["d"]
    G = Hq // Hkv
    scale = 1.0 / np.sqrt(d)
    q, kk, v, dO = (_f64(P[n]) for n in ("q", "k", "v", "dO"))
    dQ = np.zeros((T, Hq, d))
    dK = np.zeros((T, Hkv, d))
    dV = np.zeros((T, Hkv, d))
    for h in range(Hq):
        g = h // G
        M = bf.mask_from_selection([[j for j in sel[t, h] if j >= 0] for t in range(T)],
                                   P["cu"], P["B"], T)
        qt = torch.tensor(q[:, h], requires_grad=True)
        kt = torch.tensor(kk[:, g], requires_grad=True)
        vt = torch.tensor(v[:, g], requires_grad=True)
        O = torch.nn.functional.scaled_dot_product_attention(
            qt[None, None], kt[None, None], vt[None, None], attn_mask=torch.from_numpy(M)[None, None],
            scale=scale)[0, 0]
        (O * torch.from_numpy(dO[:, h])).sum().backward()
        dQ[:, h] = qt.grad.numpy()
        dK[:, g] += kt.grad.numpy()
        dV[:, g] += vt.grad.numpy()
    return dQ, dK, dV


@pytest.mark.parametrize("seed,k", [(1, 3), (2, 1), (3, 6)])
def test_matches_autograd_of_masked_attention(seed, k):
    P = _problem(seed, k=k)
    orc = _oracle(P)
    rows = _all_rows(P)
    sel, _, _ = orc.select(rows)
    dQ, dK, dV = orc.attend_backward(rows, sel, P["dO"])
    tQ, tK, tV = _torch_grads(P, sel)
    for a, b in ((dQ, tQ), (dK, tK), (dV, tV)):
        assert np.abs(a - b).max() <= 1e-12 * max(1.0, np.abs(b).max())


def test_matches_central_differences():
    P = _problem(11)
    orc = _oracle(P)
    rows = _all_rows(P)
    sel, _, _ = orc.select(rows)
    dQ, dK, dV = orc.attend_backward(rows, sel, P["dO"])
    T, Hq, Hkv, d = P["T"], P["Hq"], P["Hkv"], P["d"]
    G = Hq // Hkv
    scale = 1.0 / np.sqrt(d)
    q, kk, v, dO = (_f64(P[n]) for n in ("q", "k", "v", "dO"))
    masks = [bf.mask_from_selection([[j for j in sel[t, h] if j >= 0] for t in range(T)],
                                    P["cu"], P["B"], T) for h in range(Hq)]

    def loss(qq, k2, v2):
        tot = 0.0
        for h in range(Hq):
            O, _ = bf.masked_attention(qq[:, h], k2[:, h // G], v2[:, h // G], masks[h], scale)
            tot += float((O * dO[:, h]).sum())
        return tot

    rng = np.random.default_rng(5)
    eps = 1e-6
    for name, arr, grad in (("q", q, dQ), ("k", kk, dK), ("v", v, dV)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, n)) for n in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += eps
            minus[idx] -= eps
            args_p = {"q": q, "k": kk, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = plus, minus
            fd = (loss(args_p["q"], args_p["k"], args_p["v"]) -
                  loss(args_m["q"], args_m["k"], args_m["v"])) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


def test_sum_identities():
    P = _problem(21, k=2)
    orc = _oracle(P)
    rows = _all_rows(P)
    sel, _, _ = orc.select(rows)
    dQ, dK, dV = orc.attend_backward(rows, sel, P["dO"])
    G = P["Hq"] // P["Hkv"]
    dO = _f64(P["dO"])
    for g in range(P["Hkv"]):
        want = dO[:, g * G:(g + 1) * G].sum(axis=(0, 1))
        np.testing.assert_allclose(dV[:, g].sum(axis=0), want, rtol=0, atol=1e-11)
        np.testing.assert_allclose(dK[:, g].sum(axis=0), 0.0, rtol=0, atol=1e-11)


def test_dq_unchanged_by_a_common_key_shift():
    # integer-valued keys shifted by an integer vector stay exact in bf16
    P = _problem(31, integer=True)
    rows = _all_rows(P)
    orc = _oracle(P)
    sel, _, _ = orc.select(rows)
    dQ, _, _ = orc.attend_backward(rows, sel, P["dO"])
    c = np.random.default_rng(7).integers(-4, 5, size=P["d"]).astype(np.float32)
    shifted = _bits(_f64(P["k"]).astype(np.float32) + c[None, None, :])
    dQ2, _, _ = _oracle(P, kbits=shifted).attend_backward(rows, sel, P["dO"])
    np.testing.assert_allclose(dQ2, dQ, rtol=0, atol=1e-9)


def test_zero_output_gradient_gives_zero_gradients():
    P = _problem(41)
    rows = _all_rows(P)
    orc = _oracle(P)
    sel, _, _ = orc.select(rows)
    z = np.zeros_like(P["dO"])
    for a in orc.attend_backward(rows, sel, z):
        assert not np.any(a)
