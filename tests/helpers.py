"""Shared test plumbing: host <-> device copies of the generated inputs and the parity
tolerances. Holds none of the method's arithmetic."""

import numpy as np

# apply outputs: |y - y_ref| <= APPLY_TOL * (|y_ref| + rms(y_ref)), rms over the tensor
APPLY_TOL = 1e-2
# compress scales: relative error against the fp64 oracle
SCALE_RTOL = 1e-5


def torch():
    import torch as _t
    return _t


def dev(a, dtype=None):
    """numpy -> CUDA tensor. uint16 arrays are bf16 bit patterns, uint32 sign words go to
    int32 storage (same bits)."""
    t = torch()
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16 and dtype in (None, "bf16"):
        return t.from_numpy(a.view(np.int16)).view(t.bfloat16).cuda()
    if a.dtype == np.uint32:
        return t.from_numpy(a.view(np.int32)).cuda()
    if a.dtype == np.float16:
        return t.from_numpy(a).cuda()
    return t.from_numpy(a).cuda()


def host(tensor):
    """CUDA tensor -> numpy; bf16 -> uint16 bits, int32 sign words -> uint32."""
    t = torch()
    x = tensor.detach().cpu()
    if x.dtype == t.bfloat16:
        return x.view(t.int16).numpy().view(np.uint16)
    if x.dtype == t.int32:
        return x.numpy().view(np.uint32)
    return x.numpy()


def bf16_to_f64(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_apply_close(y, y_ref, tol=APPLY_TOL, what="y", per_token=False):
    """|y - y_ref| <= tol * (|y_ref| + rms). By default rms is over the whole output
    tensor (the stated apply tolerance). per_token=True takes the rms of each token's
    outputs (each row of a [batch, d_out] output) instead: the product is linear in each
    token's activations, so fp32 rounding of token t scales with that token's own outputs;
    the tight fp32-output checks use it so that tokens of very different magnitude are
    each held to their own scale."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    assert y.shape == y_ref.shape, (y.shape, y_ref.shape)
    if per_token and y_ref.ndim == 2 and y_ref.size:
        rms = np.sqrt(np.mean(y_ref ** 2, axis=1, keepdims=True))
    else:
        rms = np.full_like(y_ref, float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0)
    rms = np.broadcast_to(rms, y_ref.shape)
    err = np.abs(y - y_ref)
    bound = tol * (np.abs(y_ref) + rms)
    bad = err > bound
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; first at {i}: "
            f"got {y[i]!r} want {y_ref[i]!r} (rms {float(rms[i]):.3g}, max rel "
            f"{float((err / np.maximum(np.abs(y_ref) + rms, 1e-300)).max()):.3g})")


def assert_scales_close(s, s_ref, rtol=SCALE_RTOL):
    s = np.asarray(s, dtype=np.float64)
    s_ref = np.asarray(s_ref, dtype=np.float64)
    assert s.shape == s_ref.shape, (s.shape, s_ref.shape)
    err = np.abs(s - s_ref)
    bad = err > rtol * np.abs(s_ref)
    # an exactly-zero reference must be matched exactly
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"scales: {int(bad.sum())} of {bad.size} beyond {rtol} relative; first "
                             f"at {tuple(i)}: got {s[tuple(i)]!r} want {s_ref[tuple(i)]!r}")
