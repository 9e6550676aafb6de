"""Helpers for GPU tests: numpy <-> device tensors, bit comparisons."""
import numpy as np
import torch


def dev(a, dtype=None):
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def host(t):
    return t.detach().cpu().numpy()


def bits_equal(a, b):
    a = np.ascontiguousarray(a)
    b = np.ascontiguousarray(b)
    if a.dtype == np.float16:
        return np.array_equal(a.view(np.uint16), b.astype(np.float16).view(np.uint16))
    if a.dtype == np.float32:
        return np.array_equal(a.view(np.uint32), b.astype(np.float32).view(np.uint32))
    return np.array_equal(a, b)


def f16_within(y, ref, rel=1e-3, ulps=2):
    """The fp16 output contract: |y - ref| <= 1e-3 |ref| or <= 2 fp16 ulp, elementwise."""
    y = y.astype(np.float64)
    r = ref.astype(np.float64)
    ulp = np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64)
    ok = (np.abs(y - r) <= rel * np.abs(r)) | (np.abs(y - r) <= ulps * ulp) | (y == r)
    return bool(ok.all())


def ulps32(a, b):
    a = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    b = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(a - b)
