"""Helpers shared by the GPU tests: device tensors from fg_synth inputs, oracle<->device
conversions and the float tolerance (max |err| <= 1e-2 * RMS(oracle output))."""
import numpy as np

import fg_synth

TOL_RMS = 1e-2


def cuda():
    import torch
    return torch.device("cuda:0")


def to_dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(cuda())


def to_np(t):
    return t.detach().cpu().numpy()


def synth_dev(seed, stream, shape, dist="normal", scale=1.0):
    return to_dev(fg_synth.tensor(seed, stream, shape, dist, scale))


def assert_close_rms(got, ref, tol=TOL_RMS, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = float(np.max(np.abs(got - ref))) if got.size else 0.0
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert err <= tol * max(rms, 1e-30), f"{what}: max|err| {err:.3e} > {tol} * RMS {rms:.3e}"
    return err, rms
