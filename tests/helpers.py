"""Shared helpers of the GPU parity tests (test infrastructure)."""
import numpy as np
import torch

from mixture_experts_layer_counts_b200.inputs import ExpertView, host_bits
from oracle import bf16_tolerance_violation, moe_forward_ref, rel_l2

# Router weights are fp32 softmax values renormalised over the top k, from
# fp32 logits whose error is bounded by the router's certified bound; the
# induced weight error stays below this.
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


def bf16_rounding_ambiguity(inp, ref, tokens=None):
    """bf16 results of the intermediate that fp32 arithmetic can legitimately give.

    The GPU forms h = SiLU(g) * u in fp32 from fp32 tensor-core accumulators and
    rounds it once to bf16; the oracle rounds its fp64 h once.  Where the exact
    h lies closer to a bf16 rounding boundary than the kernel's fp32 arithmetic
    resolves, more than one bf16 value is a correct result.  Error band of the
    kernel's h:
        band = 2^-19 |h| + 2^-21 (|SiLU'(g) u| S_g + |SiLU(g)| S_u)
    with S_g = sum_k |x_k W1[i,k]|, S_u likewise: a few fp32 ulps of the
    accumulated magnitudes (this term dominates under cancellation, g or u
    much smaller than S) plus the SiLU's own fp32 error.  The valid results
    are the bf16 roundings of [h - band, h + band].

    Returns (amb: {perm position -> (lo, hi) arrays over I}, env [T, H]); env is
    the largest change of the output the non-nearest valid results can cause:
    env[t, o] = sum_j w[t,j] sum_i |W2[e][o, i]| * max(h_hi - r, r - h_lo).
    """
    from scipy.special import expit

    from mixture_experts_layer_counts_b200.inputs import host_bits as hb
    from oracle import bf16_bits_to_f64 as dec
    from oracle import round_to_bf16

    k = inp["top_k"]
    x = dec(hb(inp["hidden"]))
    T, H = x.shape
    perm, off, w = ref["perm"], ref["offsets"], ref["weights"]
    want = np.ones(T, bool) if tokens is None else np.isin(np.arange(T), tokens)
    amb, env = {}, np.zeros((T, H))
    for e in range(len(off) - 1):
        rows = [p for p in range(off[e], off[e + 1]) if want[perm[p] // k]]
        if not rows:
            continue
        W = dec(hb(inp["w13"][e]))
        I = W.shape[0] // 2
        Xe = x[perm[rows] // k]
        g, u = Xe @ W[:I].T, Xe @ W[I:].T
        Sg, Su = np.abs(Xe) @ np.abs(W[:I]).T, np.abs(Xe) @ np.abs(W[I:]).T
        sig = expit(g)
        s = g * sig
        ds = sig * (1.0 + g * (1.0 - sig))
        h = s * u
        r = round_to_bf16(h)
        band = 2.0 ** -19 * np.abs(h) + 2.0 ** -21 * (np.abs(ds * u) * Sg + np.abs(s) * Su)
        lo, hi = round_to_bf16(h - band), round_to_bf16(h + band)
        dev = np.maximum(hi - r, r - lo)
        W2 = None
        for ri, p in enumerate(rows):
            amb[p] = (lo[ri], hi[ri])
            a = dev[ri] > 0
            if a.any():
                W2 = dec(hb(inp["w2"][e])) if W2 is None else W2
                f = perm[p]
                env[f // k] += w[f // k, f % k] * (np.abs(W2[:, a]) @ dev[ri, a])
    return amb, env


def assert_inter_equal(dbg, ref, amb):
    """GPU intermediate == oracle intermediate wherever the rounding is unique,
    and one of the valid roundings (bf16_rounding_ambiguity) elsewhere."""
    from mixture_experts_layer_counts_b200.inputs import host_bits as hb
    from oracle import bf16_bits_to_f64 as dec

    gi = dec(hb(dbg["inter"]))
    ri = ref["inter"]
    n_amb = n_diff = 0
    for p, (lo, hi) in amb.items():
        n_diff += int((gi[p] != ri[p]).sum())
        n_amb += int((lo != hi).sum())
        ok = (gi[p] >= lo) & (gi[p] <= hi)
        assert ok.all(), f"intermediate row {p} outside its valid roundings at {np.nonzero(~ok)[0][:4]}"
    return n_diff, n_amb


# Parity records of the tests that run (written to $MOE_PARITY_LOG at the end
# of the session when that variable is set; see conftest.py).
PARITY_LOG = []


def _current_test():
    import os
    return os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]


def assert_output_close(out, ref, fp8, tokens=None, env=None):
    """Output acceptance against the oracle.

    bf16: |gpu - ref| <= 2e-2 |ref| + 2e-3 rms(ref) per element, rms over the
    compared elements.  Only a test that passes ``env`` (the output change the
    alternative correct roundings of the intermediate can cause, from
    bf16_rounding_ambiguity) may widen that bound by env, and every element
    that needed it is counted in the parity log.  FP8: relative L2 <= 3e-2.
    """
    o = out.float().cpu().numpy().astype(np.float64)
    r = ref["out"]
    if tokens is not None:
        o, r = o[tokens], r[tokens]
        env = None if env is None else env[tokens]
    if fp8:
        err = rel_l2(o, r)
        PARITY_LOG.append(dict(test=_current_test(), kind="fp8", rel_l2=err))
        assert err <= 3e-2, f"FP8 relative L2 {err:.4g} > 3e-2"
        return err
    v = bf16_tolerance_violation(o, r)
    rec = dict(test=_current_test(), kind="bf16", strict_ratio=v, n_over_strict=0, env_used=False)
    if v > 1.0 and env is not None:
        rms = float(np.sqrt(np.mean(r * r)))
        bound = 2e-2 * np.abs(r) + 2e-3 * rms
        over = np.abs(o - r) > bound
        rec.update(n_over_strict=int(over.sum()), n_elements=int(o.size), env_used=True,
                   max_env_over_bound=float((env / bound).max()),
                   ratio_with_env=bf16_tolerance_violation(o, r, extra=env))
        PARITY_LOG.append(rec)
        assert rec["ratio_with_env"] <= 1.0, f"bf16 tolerance exceeded even with the rounding envelope: {rec}"
        return v
    PARITY_LOG.append(rec)
    assert v <= 1.0, f"bf16 tolerance exceeded: worst ratio {v:.3g}"
    return v


def fp8_intermediate_check(dbg, inp, ref, s2_gpu):
    """The GPU's E4M3 intermediate codes against the oracle's h.

    The GPU forms h in fp32 from fp32 accumulations of exact E4M3 products and
    quantises fl32(h / s2) with round-to-nearest-even; where the exact h / s2
    is farther from an E4M3 rounding boundary than that arithmetic can move
    it, the code is unique and must equal E4M3(h / s2).  Band of the kernel's
    h (as in bf16_rounding_ambiguity, with a wider accumulation term for the
    long E4M3 reductions): 2^-19 |h| + 2^-17 (|SiLU'(g) u| S_g + |SiLU(g)| S_u).
    Returns (codes compared, codes that differ from E4M3(h_ref / s2_gpu),
    codes inside the ambiguous band).
    """
    from scipy.special import expit

    from mixture_experts_layer_counts_b200.inputs import host_bits as hb
    from oracle import decode_weight, e4m3_code_to_f64, round_to_e4m3_satfinite

    k = inp["top_k"]
    xq = e4m3_code_to_f64(ref["xq"]) * np.float64(ref["s1"])
    perm, off = ref["perm"], ref["offsets"]
    gi = e4m3_code_to_f64(hb(dbg["inter"]))
    s13 = inp["w13_scale"].cpu().numpy()
    n = n_diff = n_amb = 0
    for e in range(len(off) - 1):
        rows = list(range(off[e], off[e + 1]))
        if not rows:
            continue
        W = decode_weight(hb(inp["w13"][e]), s13[e])
        I = W.shape[0] // 2
        Xe = xq[perm[rows] // k]
        g, u = Xe @ W[:I].T, Xe @ W[I:].T
        Sg, Su = np.abs(Xe) @ np.abs(W[:I]).T, np.abs(Xe) @ np.abs(W[I:]).T
        sig = expit(g)
        sl = g * sig
        ds = sig * (1.0 + g * (1.0 - sig))
        h = sl * u
        band = 2.0 ** -19 * np.abs(h) + 2.0 ** -17 * (np.abs(ds * u) * Sg + np.abs(sl) * Su)
        s2 = np.float64(s2_gpu)
        c = round_to_e4m3_satfinite(h / s2)
        lo = round_to_e4m3_satfinite((h - band) / s2)
        hi = round_to_e4m3_satfinite((h + band) / s2)
        got = gi[rows]
        ok = (got >= lo) & (got <= hi)
        assert ok.all(), f"expert {e}: E4M3 intermediate codes outside their valid range"
        n += got.size
        n_diff += int((got != c).sum())
        n_amb += int((lo != hi).sum())
    PARITY_LOG.append(dict(test=_current_test(), kind="fp8_inter", codes=n, differ=n_diff, ambiguous=n_amb))
    return n, n_diff, n_amb


def assert_fp8_scales_and_codes(dbg, inp, ref):
    """s1 bit-exact, hidden_q bit-exact, s2 within the fp32 arithmetic of its
    amax, intermediate codes per fp8_intermediate_check."""
    from mixture_experts_layer_counts_b200.inputs import host_bits as hb

    sc = dbg["act_scales"].cpu().numpy()
    assert sc[0] == np.float32(ref["s1"]), "activation scale s1 differs"
    assert np.array_equal(hb(dbg["hidden_q"]), ref["xq"]), "E4M3 activation codes differ"
    rel = abs(float(sc[1]) - float(ref["s2"])) / float(ref["s2"])
    assert rel <= 2.0 ** -16, f"intermediate scale s2 {sc[1]} vs {ref['s2']}"
    return fp8_intermediate_check(dbg, inp, ref, sc[1])
