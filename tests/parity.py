"""Tolerances and comparison helpers for the GPU-versus-oracle parity tests.

bf16 path (inputs bf16, fp32 accumulation, bf16 output): max |dO| <= 1e-2,
mean |dO| <= 1e-3, max |dL| <= 1e-3 against the unrounded float64 oracle.  An
output element whose reference magnitude is so large that one bf16 ulp exceeds
1e-2 (|O| >= 2) may differ by up to that ulp instead: rounding to bf16 alone
can use half of it.  fp32 path: max |dO| <= 1e-4, max |dL| <= 1e-4.
Rows with no visible key must give exactly O = 0 and L = -inf.

e4m3 prefill (P rounded to e4m3 before P V): O within the larger of the bf16 bar and
1.5 x the distance of a rounding model of that arithmetic from the oracle; L as bf16.

Backward (bf16 gradients, P and dS rounded to bf16 before their products, outputs
rounded to bf16: each about 2^-9 relative): the forward's bar scaled by the
gradient's magnitude, max |d| <= 1e-2 * max(1, max |ref|) and
mean |d| <= 1e-3 * max(1, mean |ref|).
"""
import numpy as np

BF16_MAX_ABS = 1e-2
BF16_MEAN_ABS = 1e-3
BF16_MAX_LSE = 1e-3
F32_MAX_ABS = 1e-4
F32_MAX_LSE = 1e-4


def bf16_ulp(x):
    a = np.maximum(np.abs(x), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def compare(o_gpu, lse_gpu, o_ref, lse_ref, *, f32=False):
    """Assert the tolerances; returns a dict of the observed errors."""
    o = to_np(o_gpu) if not isinstance(o_gpu, np.ndarray) else o_gpu.astype(np.float64)
    lse = to_np(lse_gpu) if not isinstance(lse_gpu, np.ndarray) else lse_gpu.astype(np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    lse_ref = np.asarray(lse_ref, dtype=np.float64)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert lse.shape == lse_ref.shape, (lse.shape, lse_ref.shape)
    assert np.all(np.isfinite(o)), "non-finite output"
    dead = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), dead), "rows without visible keys differ"
    err = np.abs(o - o_ref)
    lerr = np.abs(lse[~dead] - lse_ref[~dead]) if np.any(~dead) else np.zeros(1)
    stats = {"max_abs": float(err.max(initial=0.0)), "mean_abs": float(err.mean()) if err.size else 0.0,
             "max_lse": float(lerr.max(initial=0.0))}
    if f32:
        assert stats["max_abs"] <= F32_MAX_ABS, stats
        assert stats["max_lse"] <= F32_MAX_LSE, stats
        return stats
    allowed = np.maximum(BF16_MAX_ABS, bf16_ulp(o_ref))
    stats["n_ulp_allowance"] = int(np.count_nonzero(err > BF16_MAX_ABS))
    assert np.all(err <= allowed), stats
    assert stats["mean_abs"] <= BF16_MEAN_ABS, stats
    assert stats["max_lse"] <= BF16_MAX_LSE, stats
    return stats


GRAD_MAX_REL = 1e-2
GRAD_MEAN_REL = 1e-3
GRAD_MODEL_FACTOR = 1.5
# every compare_grad call's errors and effective bars, printed at the end of the run
# (tests/conftest.py) so that a kernel drifting toward the model-scaled bar shows
GRAD_LOG: list = []


def bf16_backward_model(q, k, v, do, scale, causal):
    """Rounding model of the backward's stated arithmetic, for the tolerance only: the
    products of bf16 inputs accumulated in fp32, P and dS rounded to bf16 before the
    accumulating products, O and the gradients rounded to bf16.  Its distance from the
    float64 oracle is the error that arithmetic makes on these inputs; it shares nothing
    with the CUDA path.  Returns dq, dk, dv as float64 arrays in the input layouts."""
    import torch
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    out = [np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape)]
    l2e = 1.4426950408889634
    for b in range(B):
        for c in range(Hkv):
            hs = slice(c * G, (c + 1) * G)
            qf = q[b, :, hs].float().transpose(0, 1)           # [G, Sq, D]
            dof = do[b, :, hs].float().transpose(0, 1)
            kf = k[b, :, c].float()                             # [Sk, D]
            vf = v[b, :, c].float()
            s = qf @ kf.T                                       # [G, Sq, Sk]
            if causal:
                vis = torch.ones(Sq, Sk, dtype=torch.bool).tril(diagonal=Sk - Sq)
                s = s.masked_fill(~vis, float("-inf"))
            lse = torch.logsumexp(s.double() * scale, -1)
            o = torch.softmax(s.double() * scale, -1).nan_to_num(0.0) @ vf.double()
            o = o.float().bfloat16().float()
            p = torch.exp2(s * (scale * l2e) - (lse * l2e).float()[..., None]).nan_to_num(0.0)
            dsv = p * (dof @ vf.T - (dof * o).sum(-1, keepdim=True))
            pb, dsb = p.bfloat16().float(), dsv.bfloat16().float()
            dq = (scale * dsb @ kf).bfloat16().double()
            dk = (scale * (dsb.transpose(1, 2) @ qf).sum(0)).bfloat16().double()
            dv = (pb.transpose(1, 2) @ dof).sum(0).bfloat16().double()
            out[0][b, :, hs] = dq.transpose(0, 1).numpy()
            out[1][b, :, c] = dk.numpy()
            out[2][b, :, c] = dv.numpy()
    return out


def compare_grad(g_gpu, ref, model=None):
    """Assert the backward bar for one gradient tensor; returns the observed errors.
    Fixed bar: max |err| <= 1e-2 max(1, max|ref|), mean |err| <= 1e-3 max(1, mean|ref|).
    With `model` (bf16_backward_model's tensor), each bound is at least 1.5 x the
    model's own max / mean distance from the oracle: long reductions (dK, dV summed
    over G Sq rows) carry more bf16 rounding than the fixed bar allows."""
    g = to_np(g_gpu) if not isinstance(g_gpu, np.ndarray) else g_gpu.astype(np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.all(np.isfinite(g)), "non-finite gradient"
    err = np.abs(g - ref)
    big = max(1.0, float(np.abs(ref).max(initial=0.0)))
    typ = max(1.0, float(np.abs(ref).mean())) if ref.size else 1.0
    max_bar, mean_bar = GRAD_MAX_REL * big, GRAD_MEAN_REL * typ
    fixed = (max_bar, mean_bar)
    model_err = (None, None)
    if model is not None and ref.size:
        merr = np.abs(np.asarray(model, dtype=np.float64) - ref)
        model_err = (float(merr.max()), float(merr.mean()))
        max_bar = max(max_bar, GRAD_MODEL_FACTOR * model_err[0])
        mean_bar = max(mean_bar, GRAD_MODEL_FACTOR * model_err[1])
    stats = {"max_abs": float(err.max(initial=0.0)), "mean_abs": float(err.mean()) if err.size else 0.0,
             "max_bar": max_bar, "mean_bar": mean_bar, "fixed_max_bar": fixed[0],
             "fixed_mean_bar": fixed[1], "model_max": model_err[0], "model_mean": model_err[1]}
    GRAD_LOG.append(stats)
    assert stats["max_abs"] <= max_bar, stats
    assert stats["mean_abs"] <= mean_bar, stats
    return stats


def e4m3_prefill_model(q8, k8, v8, q_scale, k_scale, v_scale, scale, causal):
    """Rounding model of the e4m3 prefill, for the tolerance only: exact products of the
    decoded codes, p relative to the row max times 2^7 rounded to e4m3 (nearest even),
    O normalised by the sum of the unrounded p and rounded to bf16.  Dense layouts;
    returns O float64 like q8."""
    import torch
    f8 = torch.float8_e4m3fn

    def dec(t, sc):
        t = t.detach().cpu()
        return (t.view(f8) if t.dtype == torch.uint8 else t).to(torch.float64) * sc

    q, k, v = dec(q8, q_scale), dec(k8, k_scale), dec(v8, v_scale)
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    qt = q.permute(0, 2, 1, 3)
    kt = k.permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    vt = v.permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    s2 = (qt @ kt.transpose(-1, -2)) * (scale * 1.4426950408889634)
    if causal:
        vis = torch.ones(Sq, Sk, dtype=torch.bool).tril(diagonal=Sk - Sq)
        s2 = s2.masked_fill(~vis, float("-inf"))
    m = s2.amax(-1, keepdim=True)
    p = torch.exp2(s2 - m + 7.0).nan_to_num(0.0)
    p8 = p.float().to(f8).to(torch.float64)
    l = p.sum(-1, keepdim=True)
    o = torch.where(l > 0, (p8 @ vt) / l.clamp_min(1e-300), torch.zeros_like(qt))
    return o.to(torch.bfloat16).to(torch.float64).permute(0, 2, 1, 3).numpy()


def compare_e4m3(o_gpu, lse_gpu, o_ref, lse_ref, model):
    """The e4m3 prefill bar: O within max(fixed bar, 1.5 x the rounding model's own
    distance from the oracle), max and mean; L as the bf16 bar (L uses exact sums)."""
    o = to_np(o_gpu)
    lse = to_np(lse_gpu)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    lse_ref = np.asarray(lse_ref, dtype=np.float64)
    merr = np.abs(np.asarray(model, dtype=np.float64) - o_ref)
    err = np.abs(o - o_ref)
    max_bar = max(BF16_MAX_ABS, GRAD_MODEL_FACTOR * float(merr.max()))
    mean_bar = max(BF16_MEAN_ABS, GRAD_MODEL_FACTOR * float(merr.mean()))
    assert float(err.max()) <= max_bar, (float(err.max()), max_bar)
    assert float(err.mean()) <= mean_bar, (float(err.mean()), mean_bar)
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isneginf(lse), np.isneginf(lse_ref))
    assert float(np.abs(lse[fin] - lse_ref[fin]).max(initial=0.0)) <= BF16_MAX_LSE
    return {"max_abs": float(err.max()), "mean_abs": float(err.mean()), "max_bar": max_bar,
            "mean_bar": mean_bar}
