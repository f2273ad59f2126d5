"""The fused inverse-RoPE + per-head FP8 kernel against its oracle, through
the C ABI: codes and scales bit-exact (both sides decide the codes in the
same fp32 arithmetic), on head sizes 16..512, ragged token counts, positions
outside the table, an all-zero head, and sampled tokens of a large call."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_counts_b200 import layer
from oracle.rope_ref import inv_rope_fp8_ref

pytestmark = pytest.mark.gpu


def tables(max_pos, half, base=10000.0):
    inv = base ** (-np.arange(half) * 2.0 / (2 * half))
    ang = np.arange(max_pos)[:, None] * inv[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def run_case(T, nH, D, max_pos, seed, sample=None):
    rng = np.random.default_rng(seed)
    ct, st = tables(max_pos, D // 2)
    pos = rng.integers(0, max_pos, T).astype(np.int32)
    if T > 3:
        pos[1], pos[2] = max_pos, -5                     # no table row: codes 0, scale 0
    xt = (torch.tensor(rng.standard_normal((T, nH, D)), dtype=torch.float32) * 2).to(torch.bfloat16)
    if T > 4:
        xt[4, 0] = 0                                     # an all-zero head: scale 1, codes 0
    codes, scales = layer.inv_rope_fp8_quant(xt.cuda(), torch.from_numpy(pos).cuda(), torch.from_numpy(ct).cuda(),
                                             torch.from_numpy(st).cuda())
    torch.cuda.synchronize()
    codes, scales = codes.cpu().numpy(), scales.cpu().numpy()
    rows = np.arange(T) if sample is None else np.asarray(sample)
    rc, rs = inv_rope_fp8_ref(xt.float().numpy()[rows], pos[rows], ct, st)
    assert np.array_equal(scales[rows], rs), "scales differ"
    assert np.array_equal(codes[rows], rc), "codes differ"
    return codes, scales, pos


@pytest.mark.parametrize("T,nH,D", [(1, 1, 16), (37, 3, 64), (200, 8, 128), (5, 2, 512), (999, 4, 256),
                                    (64, 5, 32)])
def test_inv_rope_fp8_bit_exact(cuda_ok, T, nH, D):
    codes, scales, pos = run_case(T, nH, D, 4096, seed=T + nH + D)
    if T > 4:
        assert not codes[1].any() and not codes[2].any() and not scales[1].any() and not scales[2].any()
        # an all-zero head: scale 1 and codes of +0 or -0 (a zero rotated by a
        # negative sine is -0, code 0x80)
        assert scales[4, 0] == 1.0 and not (codes[4, 0] & 0x7F).any()


def test_inv_rope_fp8_large_call_sampled(cuda_ok):
    T = 16384
    rng = np.random.default_rng(0)
    sample = np.sort(np.concatenate([[0, 1, 2, T - 1], rng.choice(np.arange(3, T - 1), 60, replace=False)]))
    run_case(T, 32, 128, 8192, seed=7, sample=sample)


def e4m3_midpoints():
    """Every midpoint between neighbouring positive E4M3 values (the ties of
    its round-to-nearest-even)."""
    vals = sorted({(1 + m / 8) * 2.0 ** (e - 7) for e in range(1, 16) for m in range(8)} |
                  {m / 8 * 2.0 ** -6 for m in range(1, 8)})
    vals = [v for v in vals if v <= 448]
    mids = [(a + b) / 2 for a, b in zip(vals, vals[1:])]
    return np.array(mids)


def test_inv_rope_fp8_rounding_boundaries(cuda_ok):
    """Quotients exactly on (and next to) E4M3 ties, under scales whose
    reciprocal is inexact, and heads so small that the scale is subnormal
    (no finite reciprocal): the kernel's reciprocal path must fall back to the
    division wherever that decides the code.  Position 0 (cos 1, sin 0) keeps
    y = x exactly, so the ties reach the quantiser intact."""
    T, nH, D = 48, 4, 128
    rng = np.random.default_rng(11)
    mids = e4m3_midpoints()
    ks = [1.0, 3.0, 5.0, 7.0, 0.75, 3.0 * 2 ** -20, 5.0 * 2 ** 20]
    x = np.zeros((T, nH, D))
    for t in range(T):
        for h in range(nH):
            k = ks[(t * nH + h) % len(ks)]
            if (t * nH + h) % 11 == 10:
                k = 2.0 ** -rng.integers(128, 140)               # subnormal scale
            row = k * rng.choice(mids, D) * rng.choice([-1.0, 1.0], D)
            row[rng.integers(D)] = 448.0 * k * rng.choice([-1.0, 1.0])
            x[t, h] = row
    xt = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16)
    exact = (xt.double().numpy() == x)
    assert exact.mean() > 0.8, "too few engineered values survive the bf16 cast"
    ct, st = tables(16, D // 2)
    pos = np.zeros(T, dtype=np.int32)
    codes, scales = layer.inv_rope_fp8_quant(xt.cuda(), torch.from_numpy(pos).cuda(), torch.from_numpy(ct).cuda(),
                                             torch.from_numpy(st).cuda())
    torch.cuda.synchronize()
    rc, rs = inv_rope_fp8_ref(xt.float().numpy(), pos, ct, st)
    assert np.array_equal(scales.cpu().numpy(), rs), "scales differ"
    assert np.array_equal(codes.cpu().numpy(), rc), "codes differ"
