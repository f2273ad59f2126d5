"""Shared helpers of the GPU parity tests (test infrastructure)."""
import numpy as np
import torch

from mixture_experts_layer_counts_b200.inputs import ExpertView, host_bits
from oracle import bf16_tolerance_violation, moe_forward_ref, rel_l2

# Router weights are fp32 softmax values renormalised over the top k, from
# fp32 logits whose error is bounded by the router's certified bound; the
# induced weight error stays below this ("Router weights").
WEIGHT_ATOL = 2e-5


def custom_inputs(T, H, E, I, k, seed=0, fp8=False, bias=False, device="cuda"):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=g, device=device, dtype=torch.float32)
    d = dict(T=T, H=H, E=E, I=I, top_k=k, dtype="fp8" if fp8 else "bf16")
    d["hidden"] = r(T, H).to(torch.bfloat16)
    d["router_w"] = (r(E, H) * 0.1).to(torch.bfloat16)
    d["router_bias"] = (r(E) * 0.5) if bias else None
    w13 = r(E, 2 * I, H) * 0.02
    w2 = r(E, H, I) * 0.02
    if fp8:
        s13 = w13.abs().amax(dim=(1, 2)) / 448.0
        s2 = w2.abs().amax(dim=(1, 2)) / 448.0
        d["w13"] = (w13 / s13[:, None, None]).to(torch.float8_e4m3fn).view(torch.uint8)
        d["w2"] = (w2 / s2[:, None, None]).to(torch.float8_e4m3fn).view(torch.uint8)
        d["w13_scale"], d["w2_scale"] = s13.contiguous(), s2.contiguous()
    else:
        d["w13"], d["w2"] = w13.to(torch.bfloat16), w2.to(torch.bfloat16)
        d["w13_scale"] = d["w2_scale"] = None
    return d


def oracle_of(inp, tokens=None, keep_intermediate=False):
    fp8 = inp["dtype"] == "fp8"
    bias = None if inp["router_bias"] is None else inp["router_bias"].float().cpu().numpy()
    return moe_forward_ref(
        host_bits(inp["hidden"]), host_bits(inp["router_w"]), bias,
        ExpertView(inp["w13"]), ExpertView(inp["w2"]), inp["top_k"], inp["dtype"],
        None if not fp8 else inp["w13_scale"].cpu().numpy(),
        None if not fp8 else inp["w2_scale"].cpu().numpy(),
        tokens=tokens, keep_intermediate=keep_intermediate)


def assert_routing_equal(dbg, ref):
    ids = dbg["topk_ids"].cpu().numpy()
    assert np.array_equal(ids, ref["ids"]), "routing ids differ from the oracle"
    assert np.array_equal(dbg["counts"].cpu().numpy(), ref["counts"])
    assert np.array_equal(dbg["offsets"].cpu().numpy(), ref["offsets"])
    assert np.array_equal(dbg["perm"].cpu().numpy(), ref["perm"])
    assert np.array_equal(dbg["inv_perm"].cpu().numpy(), ref["inv_perm"])
    w = dbg["topk_w"].cpu().numpy().astype(np.float64)
    assert np.abs(w - ref["weights"]).max() <= WEIGHT_ATOL


def assert_output_close(out, ref, fp8, tokens=None):
    o = out.float().cpu().numpy().astype(np.float64)
    r = ref["out"]
    if tokens is not None:
        o, r = o[tokens], r[tokens]
    if fp8:
        err = rel_l2(o, r)
        assert err <= 3e-2, f"FP8 relative L2 {err:.4g} > 3e-2"
        return err
    v = bf16_tolerance_violation(o, r)
    assert v <= 1.0, f"bf16 tolerance exceeded: worst ratio {v:.3g}"
    return v
