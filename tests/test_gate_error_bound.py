"""CPU check of the error bound the tensor-core gate relies on.

The gate scores s~_j = fl32(mu_j * sq + acc_j) where mu_j = fl32(mean over d of Kbar_j),
r_j = Kbar_j - mu_j is held as two bf16 planes hi = bf16(r), lo = bf16(r - hi), acc_j is an fp32
accumulation of the exact bf16 products q*hi and q*lo, and sq = fl32(sum q) (sum exact in fp64).
Candidates within 2 eps of the boundary are re-scored exactly, with
    eps = 2^-11 ||q||_1 r_max + 2^-20 (|mu|_max |sum q| + max |s~|),
so the selection is exact as long as |s~ - s| <= eps. This test emulates that arithmetic in numpy
(fp32 accumulation in a random order, which bounds any fp32 summation tree) on random and
adversarial inputs (large block centres with small residuals, cancelling queries) and checks the
bound with its margin.
"""
import numpy as np
import torch


def _bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def _emulate(q, kbar, rng):
    """(s~ per block, exact s, eps) for one query row q (bf16 values) against blocks kbar [J, d]."""
    mu = kbar.mean(axis=1).astype(np.float32)                     # fp32 centres
    r = kbar - mu.astype(np.float64)[:, None]                     # exact residual of the fp32 centre
    hi = _bf16(r.astype(np.float32))
    lo = _bf16((r - hi.astype(np.float64)).astype(np.float32))
    r_max = np.float32(np.abs(r).max() * (1 + 1 / 1024))          # the pool kernel's rounded-up bound
    sq64 = q.astype(np.float64).sum()
    sq = np.float32(sq64)
    l1 = np.abs(q.astype(np.float64)).sum()
    J, d = kbar.shape
    st = np.empty(J, dtype=np.float32)
    for j in range(J):
        terms = np.concatenate([q * hi[j], q * lo[j]]).astype(np.float32)  # exact products in fp32
        acc = np.float32(0)
        for v in terms[rng.permutation(2 * d)]:
            acc = np.float32(acc + v)
        st[j] = np.float32(np.float64(mu[j]) * np.float64(sq) + np.float64(acc))  # fused multiply-add
    s = kbar @ q.astype(np.float64)
    mu_max = np.float32(np.abs(mu).max())
    eps = 2.0 ** -11 * l1 * float(r_max) + 2.0 ** -20 * (float(mu_max) * abs(sq64) + float(np.abs(st).max()))
    return st, s, eps


def test_bound_holds_with_margin_on_random_and_adversarial_rows():
    rng = np.random.default_rng(7)
    d, J = 128, 24
    worst = 0.0
    for case in range(12):
        q = _bf16(rng.normal(size=d) * (1 if case % 3 else 8))
        if case % 4 == 1:  # a cancelling query: sum q nearly 0 while ||q||_1 is large
            q = _bf16(np.concatenate([q[: d // 2], -q[: d // 2]]))
        centre = rng.normal(size=(J, 1)) * (50 if case % 2 else 0.5)  # large centres, small spread
        kbar = centre + rng.normal(size=(J, d)) * (1e-3 if case % 5 == 2 else 0.3)
        st, s, eps = _emulate(q, kbar, rng)
        err = np.abs(st.astype(np.float64) - s).max()
        assert err <= eps, (case, err, eps)
        worst = max(worst, err / eps)
    assert worst < 1 / 16, worst  # the bound is loose by more than 16x on these inputs
