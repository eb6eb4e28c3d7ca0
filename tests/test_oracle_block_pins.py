"""Pins for the oracle's encoder block on packed tokens (oracle.deit_block_cls).

The pages run attention and the MLP on the packed tokens and then extract CLS
(radpulse, "Integrated pack pipeline"; "Implications").  The oracle states one
pre-norm block in numpy float64; these pins tie it to things other than
itself:
  - torch.nn.TransformerEncoderLayer (norm_first, GELU, no biases, no dropout)
    in float64, run image by image on the surviving tokens: a separate
    implementation of the same block;
  - closed forms: zero output projections leave the CLS token unchanged;
  - invariances: the CLS row does not depend on the order of the other
    surviving tokens, nor on other images, nor on dropped tokens' values.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic

D, H, M = 96, 3, 192


def _case(seed, B=5, L=23):
    rng = synthetic.rng_for(7001, seed)
    x = rng.standard_normal((B, L, D))
    keep = (rng.random((B, L)) < 0.6).astype(np.uint8)
    w = [rng.standard_normal(s) * 0.1 for s in ((3 * D, D), (D, D), (M, D), (D, M))]
    return x, keep, w


def _torch_block(x, keep, w):
    layer = torch.nn.TransformerEncoderLayer(D, H, dim_feedforward=M, dropout=0.0, activation="gelu",
                                             batch_first=True, norm_first=True, bias=False).double().eval()
    with torch.no_grad():
        layer.self_attn.in_proj_weight.copy_(torch.from_numpy(w[0]))
        layer.self_attn.out_proj.weight.copy_(torch.from_numpy(w[1]))
        layer.linear1.weight.copy_(torch.from_numpy(w[2]))
        layer.linear2.weight.copy_(torch.from_numpy(w[3]))
        out = []
        for b in range(x.shape[0]):
            kept = keep[b] != 0
            kept[0] = True
            t = torch.from_numpy(x[b][kept])[None]
            out.append(layer(t)[0, 0].numpy())
    return np.stack(out)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_block_matches_torch_encoder_layer(seed):
    x, keep, w = _case(seed)
    got = oracle.deit_block_cls(x, keep, *w, H=H, scale=(D // H) ** -0.5)
    ref = _torch_block(x, keep, w)
    assert np.max(np.abs(got - ref)) < 1e-12


def test_block_closed_form_without_output_projections():
    x, keep, w = _case(3)
    w[1][:] = 0.0   # attention adds nothing
    w[3][:] = 0.0   # the MLP adds nothing
    got = oracle.deit_block_cls(x, keep, *w, H=H, scale=0.125)
    assert np.array_equal(got, x[:, 0])


def test_block_invariances():
    x, keep, w = _case(4)
    base = oracle.deit_block_cls(x, keep, *w, H=H, scale=0.125)
    # dropped tokens' values do not matter
    x2 = x.copy()
    x2[keep == 0] = 1e3
    x2[:, 0] = x[:, 0]
    assert np.allclose(oracle.deit_block_cls(x2, keep, *w, H=H, scale=0.125), base, rtol=0, atol=1e-12)
    # the order of the other tokens does not matter for CLS
    rng = np.random.default_rng(5)
    perm = np.concatenate([[0], 1 + rng.permutation(x.shape[1] - 1)])
    got = oracle.deit_block_cls(x[:, perm], keep[:, perm], *w, H=H, scale=0.125)
    assert np.allclose(got, base, rtol=0, atol=1e-12)
    # images are independent
    x3 = x.copy()
    x3[1:] = rng.standard_normal(x3[1:].shape)
    assert np.array_equal(oracle.deit_block_cls(x3, keep, *w, H=H, scale=0.125)[0], base[0])
