"""The intra-chunk decay factorization of the scan's output kernel, in fp32
on the CPU.

The kernel builds P[t, s] = G[t, s] exp(Acum_t - Acum_s) dt_s (s <= t) from
two factors: a column factor colf[s] = exp(Acum_r - Acum_s) dt_s, r the
first token of the 32-token block holding s, and a row factor
exp(Acum_t - Acum_r) per (row, block), both formed from the fp32 base-2
prefix a2 = log2(e) Acum.  The claims checked here:

* every factor stays finite in fp32 and their product equals the fp64 value
  to the rounding of the fp32 prefix, even under the heaviest decay of the
  synthetic inputs (A = -16, dt = 0.1 on every token) and on a ragged chunk;
  only terms below 1e-20 of the diagonal's may flush to zero (the row factor
  leaves fp32 range first);
* the head-independent alternative (one reference per chunk, the factors
  folded into the operands) leaves fp32 range under that decay, which is why
  the kernel does not use it."""
import numpy as np
import pytest

LOG2E = np.float32(1.4426950408889634)


def _decay_terms(dt, A):
    """fp32 prefix and the two factors, as the kernel forms them."""
    a2 = np.cumsum((dt * A).astype(np.float32), dtype=np.float32) * LOG2E
    r0 = (np.arange(len(dt)) // 32) * 32
    colf = np.exp2(a2[r0] - a2).astype(np.float32) * dt.astype(np.float32)
    return a2, colf, r0


@pytest.mark.parametrize("S,heavy", [(256, False), (256, True), (201, True), (128, True)])
def test_block_factors_are_finite_and_exact(S, heavy):
    r = np.random.default_rng(S + heavy)
    A = np.float32(-16.0) if heavy else np.float32(-np.exp(r.uniform(0, np.log(16))))
    dt = (np.full(S, 0.1) if heavy else np.exp(r.uniform(np.log(1e-3), np.log(1e-1), S))).astype(np.float32)
    a2, colf, r0 = _decay_terms(dt, A)
    assert np.all(np.isfinite(colf)) and np.all(colf > 0)
    acum64 = np.cumsum(dt.astype(np.float64) * float(A))
    for t in range(S):
        s = np.arange(t + 1)
        rf = np.exp2(a2[t] - a2[r0[s]]).astype(np.float32)     # row factor of each column's block
        assert np.all(np.isfinite(rf)) and np.all(rf <= 1.0)
        got = (colf[s] * rf).astype(np.float64)
        want = np.exp(acum64[t] - acum64[s]) * dt[s]
        # the row factor underflows fp32 only for terms below about 2^-75 dt of
        # the diagonal's; those may come out 0 (they are far below any output's
        # rounding)
        normal = want > 1e-20 * dt[t]
        # each fp32 addition between s and t rounds the exponent by at most half
        # an ulp of |Acum_t|, and exp2 turns that into the same relative error
        tol = 1e-6 + (t - s + 2) * np.abs(acum64[t]) * 2.0 ** -23
        assert np.all(np.abs(got[normal] - want[normal]) <= (tol * want)[normal]), t
        assert np.all(got[~normal] <= 1e-20 * dt[t])


def test_head_independent_split_leaves_fp32_range():
    S, A = 256, np.float32(-16.0)
    dt = np.full(S, 0.1, dtype=np.float32)
    a2 = np.cumsum((dt * A).astype(np.float32), dtype=np.float32) * LOG2E
    # one reference per chunk: x_s scaled by exp(-Acum_s) dt_s, y_t by exp(Acum_t)
    with np.errstate(over="ignore"):
        col = np.exp2(-a2).astype(np.float32)
    assert not np.all(np.isfinite(col))
    assert float(-a2[-1] / LOG2E) > 400   # the factors span exp(+-400) over the chunk
