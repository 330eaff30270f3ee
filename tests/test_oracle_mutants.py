"""Plant plausible mistakes in copies of the oracle source and check that the
pins catch every one of them.  Each mutant is compiled from a modified copy of
``oracle/dart_oracle.c`` in a temporary directory; the real oracle is never
touched.  Every mutation keeps all memory accesses inside the buffers."""
import os

import pytest

from oracle import dart_oracle
from tests import oracle_pins

# (name, text to find, replacement, which occurrence: 0-based)
MUTATIONS = [
    ("input_drops_dt", "const double inp = dtt * (double)Bt[n] * (double)xt[p];",
     "const double inp = (double)Bt[n] * (double)xt[p];", 0),
    ("decay_sign", "const double decay = exp(dtt * Ah);", "const double decay = exp(-0.5 * dtt * Ah);", 0),
    ("decay_after_input", "Hs[n * P + p] = decay * Hs[n * P + p] + inp;",
     "Hs[n * P + p] = decay * (Hs[n * P + p] + inp);", 0),
    ("readout_uses_B", "for (int n = 0; n < N; ++n) acc += (double)Ct[n] * Hs[n * P + p];",
     "for (int n = 0; n < N; ++n) acc += (double)Bt[n] * Hs[n * P + p];", 0),
    ("no_chunk_reset", "if (t % S == 0) memset(D, 0, sizeof(double) * (size_t)N * P);", "", 0),
    ("memory_not_decayed", "D[n * P + p] = decay * D[n * P + p] + inp;",
     "D[n * P + p] = D[n * P + p] + inp;", 0),
    ("states_from_memory", "if (c->states) memcpy(c->states + off, Hs,",
     "if (c->states) memcpy(c->states + off, D,", 0),
    ("x_wrong_head", "const float* xt = c->x + (((size_t)b * L + t) * H + h) * P;",
     "const float* xt = c->x + (((size_t)b * L + t) * H + 0) * P;", 0),
    ("mask_off_by_one", "const int k = t / S; /* chunk holding t; memories are c < k */",
     "const int k = (t + 1) / S;", 0),
    ("scale_by_P", "const double inv_sqrt_n = 1.0 / sqrt((double)N);",
     "const double inv_sqrt_n = 1.0 / sqrt((double)P);", 0),
    ("value_read_with_Q", "for (int n = 0; n < N; ++n) acc += (double)Ct[n] * M[n * P + p];",
     "for (int n = 0; n < N; ++n) acc += (double)Qt[n] * M[n * P + p];", 0),
    ("key_transposed_index", "for (int p = 0; p < P; ++p) acc += M[n * P + p] * (double)Et[p];",
     "for (int p = 0; p < P; ++p) acc += M[(n * P + p) % N * P + p % N] * (double)Et[p];", 0),
    ("softmax_unnormalised", "const double w = exp(sc[cc] - m) / z;", "const double w = exp(sc[cc] - m);", 0),
    ("gate_convex", "c->y[row + p] = base + c->g * o[p];",
     "c->y[row + p] = (1.0 - c->g) * base + c->g * o[p];", 0),
    ("gate_ignored", "c->y[row + p] = base + c->g * o[p];", "c->y[row + p] = base + o[p];", 0),
    ("decode_memory_not_decayed", "D[n * P + p] = decay * D[n * P + p] + inp;",
     "D[n * P + p] = D[n * P + p] + inp;", 1),
    ("decode_sees_open_chunk", "const int nmem = c->nchunks[b];",
     "const int nmem = c->nchunks[b] + (c->pos[b] == S - 1);", 0),
    ("decode_no_reset_after_append", "memset(D, 0, sizeof(double) * (size_t)N * P);\n        if (c->memlog)",
     "if (c->memlog)", 0),
    ("decode_gate_dropped", "yt[p] += c->g * acc;", "yt[p] += acc;", 0),
    ("partial_chunk_not_closed", "if (t % S == S - 1 || t == L - 1) {", "if (t % S == S - 1) {", 0),
    ("sma_memory_stride_floor", "const int nchunks = (L + S - 1) / S;\n    const int b = unit / H, h = unit % H;\n    const int nrows",
     "const int nchunks = L / S;\n    const int b = unit / H, h = unit % H;\n    const int nrows", 0),
    ("decay_window_from_e", "for (int r = ec + 1; r <= t; ++r)", "for (int r = ec; r <= t; ++r)", 0),
    ("decay_window_before_t", "for (int r = ec + 1; r <= t; ++r)", "for (int r = ec + 1; r < t; ++r)", 0),
    ("decay_value_only", "key[n] = wdec * acc;", "key[n] = acc;", 0),
    ("decay_key_only", "val[(size_t)cc * P + p] = wdec * acc;", "val[(size_t)cc * P + p] = acc;", 0),
    ("decay_wrong_head", "(double)c->dt[((size_t)b * L + r) * H + h] * (double)c->A[h];",
     "(double)c->dt[((size_t)b * L + r) * H + h] * (double)c->A[0];", 0),
    ("decay_sign_flipped", "wdec = exp(logdec);", "wdec = exp(-logdec);", 0),
    ("decode_memlog_after_use", "*lw += dtt * (double)c->A[h]; /* now sum_{r=e(c)+1}^{t} dt_r A_h */\n                wdec = exp(*lw);",
     "wdec = exp(*lw);\n                *lw += dtt * (double)c->A[h];", 0),
    ("decode_memlog_not_reset", "if (c->memlog) c->memlog[bh * (size_t)c->cmax + nmem] = 0.0;", "", 0),
    ("decode_decay_value_only", "key[n] = wdec * acc;", "key[n] = acc;", 1),
    ("e4m3_truncates", "double q = nearbyint(ldexp(a, 3 - E));", "double q = floor(ldexp(a, 3 - E));", 0),
    ("e4m3_row_exponent_too_big", "int k = f <= 0.875 ? e - 9 : e - 8;", "int k = e - 8;", 0),
    ("e4m3_sign_dropped", "return sign | (uint8_t)(code > 0x7E ? 0x7E : code);",
     "return (uint8_t)(code > 0x7E ? 0x7E : code);", 0),
    ("e4m3_subnormal_step", "const double q = nearbyint(a * 512.0);", "const double q = nearbyint(a * 256.0);", 0),
    ("e4m3_decode_bias", "ldexp(8.0 + m, e - 10)", "ldexp(8.0 + m, e - 11)", 0),
    ("decode_append_not_quantized", "if (c->cache_e4m3) {", "if (0) {", 0),
    ("group_by_modulo", "return h / (d->nheads / ngroups_of(d));", "return h % ngroups_of(d);", 0),
    ("bwd_memory_gradient_ignored", "K[i] = c->gD ? c->gD[(((size_t)b * H + h) * nchunks + ck) * NP + i] : 0.0;",
     "K[i] = 0.0;", 0),
    ("bwd_memory_gradient_wrong_chunk", "c->gD[(((size_t)b * H + h) * nchunks + ck) * NP + i]",
     "c->gD[(((size_t)b * H + h) * nchunks + (ck + 1) % nchunks) * NP + i]", 0),
    ("bwd_dC_from_previous_state", "sc += hcur[n * P + p] * dyt[p];", "sc += hprev[n * P + p] * dyt[p];", 0),
    ("bwd_decay_grad_drops_memory_term",
     "da += G[n * P + p] * hprev[n * P + p] + K[n * P + p] * dprev[n * P + p];",
     "da += G[n * P + p] * hprev[n * P + p];", 0),
    ("bwd_dx_without_dt", "c->dx[(TOK(t) * H + h) * P + p] = dtt * s;", "c->dx[(TOK(t) * H + h) * P + p] = s;", 0),
    ("bwd_dinit_one_decay_short", "for (int i = 0; i < NP; ++i) {\n                G[i] *= a;",
     "for (int i = 0; i < NP; ++i) {\n                if (t > 0) G[i] *= a;", 0),
]


def _mutate(src, old, new, occ):
    idx = -1
    for _ in range(occ + 1):
        idx = src.find(old, idx + 1)
        assert idx >= 0, f"pattern not found: {old!r}"
    return src[:idx] + new + src[idx + len(old):]


@pytest.mark.parametrize("name,old,new,occ", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutant_is_caught(tmp_path, name, old, new, occ):
    with open(dart_oracle.SOURCE) as f:
        src = f.read()
    mutated = _mutate(src, old, new, occ)
    assert mutated != src
    csrc = os.path.join(tmp_path, f"mut_{name}.c")
    with open(csrc, "w") as f:
        f.write(mutated)
    lib = dart_oracle.build(csrc, os.path.join(tmp_path, f"libmut_{name}.so"))
    orc = dart_oracle.Oracle(lib, nthreads=2)
    failures = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            failures.append(pin.__name__)
    assert failures, f"mutation {name} was not caught by any pin"
