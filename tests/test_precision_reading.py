"""The arithmetic behind the attention parity bound (design reading R22), on
CPU: probabilities rounded to bf16 once before P.V, binary32 softmax and
sums, bf16 output, against the float64 definition of attention rounded to
bf16.  Every output stays within one bf16 unit in the last place of the
definition's value plus 2^-9, and at least half are identical: the bound the
GPU attention tests apply."""
import numpy as np


def _bf16(x):
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    return (((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16).astype(np.uint32).view(np.float32)


def test_single_bf16_probabilities_stay_within_one_ulp_plus_2_pow_minus_9():
    rng = np.random.default_rng(22)
    D = 256
    same = total = 0
    worst = -1.0
    for n_keys in (130, 700, 2500, 4000):
        for _ in range(4):
            q = _bf16(rng.standard_normal((40, D)))
            K = _bf16(rng.standard_normal((n_keys, D)))
            V = _bf16(rng.standard_normal((n_keys, D)))
            s = (q.astype(np.float64) @ K.T.astype(np.float64)) / np.sqrt(D)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            want = _bf16((p @ V.astype(np.float64)) / p.sum(axis=1, keepdims=True)).astype(np.float64)
            # the kernel's scheme: log2-domain binary32 scores, p = 2^(s - m),
            # P rounded to bf16 for P.V, row sums of the unrounded p
            sl = (q @ K.T).astype(np.float32) * np.float32(1.4426950408889634 / np.sqrt(D))
            pf = np.exp2(sl - sl.max(axis=1, keepdims=True)).astype(np.float32)
            got = _bf16((_bf16(pf) @ V) / pf.sum(axis=1, keepdims=True)).astype(np.float64)
            ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(want), 2.0 ** -126))) - 7)
            worst = max(worst, float((np.abs(got - want) - ulp).max()))
            same += int(np.sum(got == want))
            total += got.size
    assert worst <= 2.0 ** -9, worst
    assert same / total >= 0.5, same / total
