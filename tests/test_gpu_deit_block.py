"""A random-weight DeiT-S encoder block on packed tokens, against the fp64 oracle.

The pages put the wall-clock gain of pruning in the layers that run on the
packed tokens (radpulse, "Integrated pack pipeline"; "Implications").  Here
the block is ragged_pack -> LayerNorm -> QKV -> ragged_attn_fwd -> projection
-> residual -> LayerNorm -> MLP (GELU) -> residual -> CLS rows, in f16 with
torch's GEMMs, and oracle.deit_block_cls states the same block in float64.

Bound: the f16 path rounds ten intermediate tensors on the way to a CLS
element (LN1, QKV, attention, projection, first residual, LN2, W1, GELU, W2,
second residual).  Each rounding is at most half a unit in the last place of
a value below 8 in magnitude (2^-10 = 9.8e-4 on [4, 8)), and the linears
(weights N(0, 0.02^2), fan-in 384 or 1536) shrink an input error rather than
grow it (0.02 * sqrt(1536) < 1), so the sum of the ten, 2e-2, bounds the
error in the worst alignment.  The test asserts it and also that the typical
(RMS) error stays at the size of one rounding.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import ragged_variable_length_b200 as rv
import synthetic

pytestmark = pytest.mark.gpu

D, H, d, M, L_full = 384, 6, 64, 1536, 197


def _weights(rng):
    return [(rng.standard_normal(s) * 0.02).astype(np.float16) for s in ((3 * D, D), (D, D), (M, D), (D, M))]


@pytest.mark.parametrize("B,rate", [(32, 0.5), (8, 0.0)])
def test_packed_block_matches_oracle(B, rate):
    rng = synthetic.rng_for(5003, B * 10 + int(rate * 10))
    lengths = synthetic.serving_lengths(rng, B, rate)
    keep_np = synthetic.topk_keep_mask(rng, L_full, lengths)
    x_np = rng.standard_normal((B, L_full, D)).astype(np.float16)
    w_np = _weights(rng)
    Wqkv, Wo, W1, W2 = (torch.from_numpy(w).cuda() for w in w_np)
    x = torch.from_numpy(x_np).cuda()
    keep = torch.from_numpy(keep_np).cuda()
    T = int(lengths.sum())

    xp, cu = rv.ragged_pack(x, keep)
    h = xp[:T]
    qkv = F.linear(F.layer_norm(h, (D,)), Wqkv).view(T, 3, H, d)
    a = rv.ragged_attn_fwd(qkv[:, 0], qkv[:, 1], qkv[:, 2], cu, L_full, 0.125).view(T, D)
    h = h + F.linear(a, Wo)
    h = h + F.linear(F.gelu(F.linear(F.layer_norm(h, (D,)), W1)), W2)
    cls = h[cu[:-1].long()].double().cpu().numpy()
    torch.cuda.synchronize()
    assert rv.ragged_get_device_status() == 0

    ref = oracle.deit_block_cls(x_np, keep_np, *w_np, H=H, scale=0.125)
    err = np.abs(cls - ref)
    assert float(np.max(np.abs(ref))) < 8.0
    assert float(err.max()) <= 2e-2, f"max abs error {err.max():.3e}"
    assert float(np.sqrt(np.mean(err ** 2))) <= 1e-3, f"rms error {np.sqrt(np.mean(err ** 2)):.3e}"
