"""The seeded input generator: determinism, counter addressing, rounding and the workload's distribution."""
import numpy as np
import torch

import synth


def test_bf16_rounding_is_rne():
    xs = np.random.default_rng(0).normal(size=20000).astype(np.float32).astype(np.float64)
    got = np.array([synth.bf16_rne(x) for x in xs], dtype=np.uint16)
    want = torch.from_numpy(xs.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    np.testing.assert_array_equal(got, want)
    assert synth.bf16_rne(1.0 + 2.0 ** -8) == 0x3F80          # halfway, even neighbour 1.0
    assert synth.bf16_rne(1.0 + 3 * 2.0 ** -8) == 0x3F82      # halfway, even neighbour 1 + 2^-6
    assert synth.bf16_rne(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81  # just above halfway


def test_counter_addressing_and_determinism():
    a = synth.normal(7, synth.Q_ID, (1000,))
    b = synth.normal(7, synth.Q_ID, (10,))
    assert torch.equal(a[:10], b)
    assert torch.equal(a, synth.normal(7, synth.Q_ID, (1000,)))
    assert not torch.equal(a, synth.normal(8, synth.Q_ID, (1000,)))
    assert not torch.equal(a, synth.normal(7, synth.V_ID, (1000,)))
    assert synth.bf16_rne(synth.normal_at(7, synth.Q_ID, 5)) == int(a[5].view(torch.int16).item()) & 0xFFFF


def test_normal_moments():
    x = synth.normal(3, synth.V_ID, (1 << 20,)).double()
    assert abs(x.mean().item()) < 0.005
    assert abs(x.std().item() - 1.0) < 0.005
    assert abs(((x ** 4).mean() / x.var() ** 2).item() - 3.0) < 0.05  # Gaussian kurtosis


def test_key_block_offsets():
    B, N, Hkv, d, bs = 2, 2048, 2, 128, 256
    k = synth.keys(5, B, N, Hkv, d, bs).double()
    nblk = N // bs
    means = k.reshape(B, nblk, bs, Hkv, d).mean(dim=(2, 4))  # [B, nblk, Hkv]
    offs = torch.tensor([[[synth.key_offset(5, b, h, j, Hkv, nblk) for h in range(Hkv)] for j in range(nblk)]
                         for b in range(B)], dtype=torch.float64)
    assert (means - offs).abs().max().item() < 0.02  # noise of a mean over 32768 N(0,1) values
    assert 0.3 < offs.std().item() < 0.8             # offsets ~ N(0, 0.5^2)
