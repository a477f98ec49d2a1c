"""Shared helpers of the GPU parity tests: run the CUDA path and the float64
oracle on the same seeded inputs and compare them."""
import numpy as np
import torch

import oracle
import workloads

# max-abs error allowed against the unrounded float64 oracle (fp32 accumulation)
TOLERANCE = {"fp16": 2e-3, "bf16": 1.5e-2}

# Selective GEMM: the kernel rounds the hidden activations and the output to the
# input dtype, the oracle keeps both in float64.  Rounding the output costs at
# most half an ulp, u*|y| (u = 2^-11 fp16, 2^-8 bf16); rounding the hidden
# activations adds an error of standard deviation about u/sqrt(3) * sqrt(sum_t
# h_t^2 W2[t,c]^2) ~ u/sqrt(3) for these inputs, which TOLERANCE bounds at 6 sigma.
MLP_RTOL = {"fp16": 2.0 ** -11, "bf16": 2.0 ** -8}


def mlp_excess(got, want, dtype):
    """Largest amount by which |got - want| exceeds TOLERANCE + MLP_RTOL * |want|
    (<= 0 passes), and the max-abs error."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    diff = np.abs(got - want)
    bound = TOLERANCE[dtype] + MLP_RTOL[dtype] * np.abs(want)
    return float((diff - bound).max()), float(diff.max())


def active_mask(idx, B, H_kv, G):
    """bool [B, H_q]: query rows the call must write."""
    mask = np.zeros((B, H_kv * G), dtype=bool)
    for b, row in enumerate(np.asarray(idx)):
        for h in row:
            if 0 <= h < H_kv:
                mask[b, h * G:(h + 1) * G] = True
    return mask


def sentinel_bits(dtype):
    return np.uint16(workloads.SENTINEL[dtype])


def out_bits(out):
    return out.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def as_f64(out):
    return out.detach().cpu().double().numpy()


def check_against_oracle(w, q, k, v, idx, out_gpu, expected=None):
    """Elementwise parity over every active row, bit-exact sentinel elsewhere.
    q/k/v/idx may live on the GPU; they are copied to the host for the oracle.
    Returns the max-abs error."""
    idx_h = idx.cpu().numpy()
    if expected is None:
        expected, _ = oracle.sha_decode(q.cpu(), k.cpu(), v.cpu(), idx_h, w.scale, w.dtype)
    mask = active_mask(idx_h, w.B, w.H_kv, w.G)
    bits = out_bits(out_gpu).reshape(w.B, w.H_q, w.d)
    assert (bits[~mask] == sentinel_bits(w.dtype)).all(), "an inactive row was written"
    got = as_f64(out_gpu).reshape(w.B, w.H_q, w.d)
    err = np.abs(got[mask] - expected[mask]).max() if mask.any() else 0.0
    assert np.isfinite(got[mask]).all(), "non-finite output in an active row"
    assert err <= TOLERANCE[w.dtype], f"max-abs error {err} > {TOLERANCE[w.dtype]}"
    return float(err)


def sampled_units(w, idx, n_random, seed=0):
    """(b, h) pairs to check one by one: every unit of the first and last batch
    row plus n_random others drawn with a seeded generator."""
    idx_h = idx.cpu().numpy()
    rng = np.random.default_rng(seed)
    picks = {(0, int(h)) for h in idx_h[0]} | {(w.B - 1, int(h)) for h in idx_h[-1]}
    for u in rng.choice(w.B * w.top_k, size=min(n_random, w.B * w.top_k), replace=False):
        b, kk = divmod(int(u), w.top_k)
        picks.add((b, int(idx_h[b, kk])))
    return sorted(picks)


def check_sampled_units(w, q, k, v, idx, out_gpu, n_random=32, seed=0):
    """Full-size parity: the sentinel over the whole output (bit-exact) and the
    oracle on sampled units, gathered to the host one by one."""
    idx_h = idx.cpu().numpy()
    mask = active_mask(idx_h, w.B, w.H_kv, w.G)
    bits = out_bits(out_gpu).reshape(w.B, w.H_q, w.d)
    assert (bits[~mask] == sentinel_bits(w.dtype)).all(), "an inactive row was written"
    got = as_f64(out_gpu).reshape(w.B, w.H_q, w.d)
    assert np.isfinite(got[mask]).all()
    units = sampled_units(w, idx, n_random, seed)
    G = w.G
    qu = torch.stack([q[b, h * G:(h + 1) * G].cpu() for b, h in units])
    ku = torch.stack([k[b, h].cpu() for b, h in units])
    vu = torch.stack([v[b, h].cpu() for b, h in units])
    ref = oracle.sha_units(qu, ku, vu, w.scale, w.dtype)
    err = 0.0
    for i, (b, h) in enumerate(units):
        err = max(err, float(np.abs(got[b, h * G:(h + 1) * G] - ref[i]).max()))
    assert err <= TOLERANCE[w.dtype], f"max-abs error {err} > {TOLERANCE[w.dtype]}"
    return err, len(units)
