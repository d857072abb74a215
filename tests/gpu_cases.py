"""Shared helpers of the GPU parity tests: seeded cases, oracle comparison."""
import numpy as np
import torch

from sparse_weight_b200 import hyb, inputs

TOL = 2e-3  # |y - y_ref| <= TOL * (|W_hat| |x| + |U| (|V|^T |x|)), fp32 accumulation


def dev():
    return torch.device("cuda:0")


def case(n, k, b1, b2, tmap, batch=1, std=0.02, outliers=0.0, name="case", rank=0,
         lr_std=0.01):
    """Seeded bf16 weight, map, activations (and low-rank factors)."""
    W = inputs.weight(n, k, std, inputs.seed_of(name, n, k, "W"), outliers=outliers)
    X = inputs.activations(batch, k, inputs.seed_of(name, n, k, "X", batch))
    UV = inputs.lowrank(n, k, rank, lr_std, inputs.seed_of(name, n, k, "LR")) if rank else None
    return W, np.asarray(tmap, np.uint8), X, UV


def packed_to_host(P: hyb.Packed):
    return dict(vals=P.vals.cpu().numpy().view(np.uint16),
                meta=P.meta.cpu().numpy()[:P.n_meta],
                val_off=P.val_off.cpu().numpy(),
                meta_off=P.meta_off.cpu().numpy())


def assert_pack_equal(P: hyb.Packed, ref):
    got = packed_to_host(P)
    for key in ("val_off", "meta_off", "vals", "meta"):
        a, b = got[key], ref[key]
        assert a.shape == b.shape, (key, a.shape, b.shape)
        if not np.array_equal(a, b):
            bad = np.nonzero(a != b)[0]
            raise AssertionError(f"{key}: {bad.size} mismatches, first at {bad[:5]}: "
                                 f"got {a[bad[:5]]} want {b[bad[:5]]}")


def assert_within(y, y_ref, env, tol=TOL, what=""):
    y = np.asarray(y, np.float64)
    err = np.abs(y - y_ref)
    bound = tol * env
    ok = err <= bound
    if not ok.all():
        idx = np.argwhere(~ok)[:5]
        raise AssertionError(f"{what}: {int((~ok).sum())} outputs outside tolerance, e.g. "
                             + ", ".join(f"{tuple(i)} got {y[tuple(i)]!r} want "
                                         f"{y_ref[tuple(i)]!r} bound {bound[tuple(i)]!r}"
                                         for i in idx))


def bf16_within_one_ulp(y_bf16: torch.Tensor, y_f32: torch.Tensor):
    """bf16 output equals the round-to-nearest-even of the fp32 output (<= 1 ulp)."""
    a = y_bf16.view(torch.int16).to(torch.int32).cpu()
    b = y_f32.to(torch.bfloat16).view(torch.int16).to(torch.int32).cpu()
    assert (a - b).abs().max().item() <= 1
