"""Closed-form inputs of the golden fixtures (no part of the method).

Every value is a small multiple of 1/8, exactly representable in bf16, so
the oracle and the CUDA path read identical inputs.  Rows of some keys are
boosted so that the pooled scores have clear margins at the k-th place."""
import numpy as np


def tensor(shape, a, c, m, scale=8.0):
    """x[flat] = (((flat * a + c) * 2654435761 mod 2^32) >> 8 mod m - m // 2) / scale"""
    n = int(np.prod(shape))
    flat = np.arange(n, dtype=np.uint64)
    h = ((flat * np.uint64(a) + np.uint64(c)) * np.uint64(2654435761)) % np.uint64(1 << 32)
    x = ((h >> np.uint64(8)) % np.uint64(m)).astype(np.int64) - m // 2
    return (x.astype(np.float64) / scale).reshape(shape)


def case(spec):
    """(q, k, v) of one fixture spec: dict with B, Hq, Hkv, d, N, q_len and
    the generator constants; keys listed in `boost` get +1 on every dim of
    head 0's query direction (a planted salient set)."""
    B, Hq, Hkv, d, N, L = spec["B"], spec["Hq"], spec["Hkv"], spec["d"], spec["N"], spec["q_len"]
    q = tensor((B, Hq, L, d), *spec["q_gen"])
    k = tensor((B, Hkv, N, d), *spec["k_gen"])
    v = tensor((B, Hkv, N, d), *spec["v_gen"])
    for j in spec.get("boost", []):
        k[:, :, j, :] += np.sign(q[:, 0:1, 0, :]) * 0.5
    return q, k, v
