"""GPU parity of the Mamba-2 block steps either side of the SSD (causal conv1d + SiLU,
gated RMSNorm) against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import ssd_sequence_mixing_b200 as ssd
from harness import assert_close

pytestmark = pytest.mark.gpu

DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def seeded(shape, seed, scale=1.0):
    return torch.from_numpy(np.random.default_rng(seed).standard_normal(shape) * scale)


@pytest.mark.parametrize("case", [
    # batch, seqlen, channels, dtype, lengths (packed) or None, bias
    (2, 300, 5376 // 16, "bf16", None, True),
    (3, 70, 40, "f32", None, False),
    (1, 0, 64, "bf16", [1, 2, 0, 3, 130, 64, 65, 0, 5], True),
    (1, 0, 5376, "bf16", [2048, 1000, 1048], True),
    (4, 2, 8, "f32", None, True),
], ids=["bf16_dense", "f32_dense", "bf16_packed_short", "bf16_mamba_channels", "f32_shorter_than_window"])
def test_causal_conv1d_silu(case):
    batch, T, ch, dtype, lengths, with_bias = case
    if lengths is not None:
        T = sum(lengths)
    x = seeded((batch, T, ch), 1).to(DT[dtype])
    w = seeded((ch, 4), 2, 0.5).float()
    b = seeded((ch,), 3, 0.1).float() if with_bias else None
    cu = None
    if lengths is not None:
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32)
    out = ssd.causal_conv1d_silu(x.cuda(), w.cuda(), None if b is None else b.cuda(),
                                 None if cu is None else cu.cuda())
    torch.cuda.synchronize()
    for r in range(batch):
        offs = None if cu is None else cu.numpy()
        ref = oracle.causal_conv1d_silu(x[r].double().numpy(), w.double().numpy(),
                                        None if b is None else b.double().numpy(), offs)
        assert_close(f"conv row {r}", out[r].float().cpu().numpy(), ref, dtype)


@pytest.mark.parametrize("case", [(2048, 5120, "bf16"), (300, 64, "f32"), (17, 8, "bf16"), (5, 8192, "f32")],
                         ids=["bf16_mamba_dim", "f32_small", "bf16_tiny", "f32_max_dim"])
def test_gated_rmsnorm(case):
    tokens, dim, dtype = case
    y = seeded((tokens, dim), 4).to(DT[dtype])
    z = seeded((tokens, dim), 5).to(DT[dtype])
    w = (1.0 + seeded((dim,), 6, 0.1)).float()
    out = ssd.gated_rmsnorm(y.cuda(), z.cuda(), w.cuda(), eps=1e-5)
    torch.cuda.synchronize()
    ref = oracle.gated_rmsnorm(y.double().numpy(), z.double().numpy(), w.double().numpy(), eps=1e-5)
    assert_close("gated rmsnorm", out.float().cpu().numpy(), ref, dtype)
