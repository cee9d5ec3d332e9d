"""Planted mistakes in the oracle must be caught by the pins.

Each case copies the oracle's C source, applies one plausible mistake (a
dropped term, a wrong sign, a wrong constant, an off-by-one bound, a swapped
bit order), compiles the copy on the CPU and runs the pin checks against it.
At least one pin must fail for every mutant; this shows that the pins
constrain every part of the oracle rather than echoing it.
"""
import os

import pytest

from oracle import pq_oracle
from tests import oracle_pins

MUTANTS = {
    "seq2_shift": ("p->kh = 2.0f; p->shift = 0.5f;",
                   "p->kh = 2.0f; p->shift = 0.25f;"),
    "clip_at_one": ("const float clip_seq = 0.99f;",
                    "const float clip_seq = 1.0f;"),
    "round_half_up": ("r = nearbyintf(t);", "r = floorf(t + 0.5f);"),
    "lsq_round_half_up": ("r = nearbyintf(xc);", "r = floorf(xc + 0.5f);"),
    "dalpha_sign": ("((double)lev - (inside ? (double)x : 0.0))",
                    "((double)lev + (inside ? (double)x : 0.0))"),
    "dalpha_drop_x": ("((double)lev - (inside ? (double)x : 0.0))",
                      "((double)lev)"),
    "dalpha_drop_level": ("((double)lev - (inside ? (double)x : 0.0))",
                          "(0.0 - (inside ? (double)x : 0.0))"),
    "dalpha_no_mask": ("((double)lev - (inside ? (double)x : 0.0))",
                       "((double)lev - (double)x)"),
    "ste_open_interval": ("*inside = (x >= p.lo) && (x <= p.hi);",
                          "*inside = (x > p.lo) && (x < p.hi);"),
    "ste_no_gate": ("dw[r * cols + j] = inside ? g : 0.0f;",
                    "dw[r * cols + j] = g;"),
    "pack_bit_order": ("<< (p.bits * slot)",
                       "<< (p.bits * (int)(per_byte - 1 - slot))"),
    "bf16_round_half_up": ("u += 0x7FFFu + ((u >> 16) & 1u);", "u += 0x8000u;"),
    "bf16_truncate": ("u += 0x7FFFu + ((u >> 16) & 1u);", "u += 0u;"),
    "lsq_hi_bound": ("p->lo = -half; p->hi = half - 1.0f;",
                     "p->lo = -half; p->hi = half;"),
    "ternary_shift": ("p->lo = -clip_seq; p->hi = clip_seq; p->kh = 1.5f; p->shift = 0.0f;",
                      "p->lo = -clip_seq; p->hi = clip_seq; p->kh = 1.5f; p->shift = 0.5f;"),
    "grad_scale_no_sqrt": ("(float)(1.0 / sqrt((double)cols * (double)p.qp))",
                           "(float)(1.0 / ((double)cols * (double)p.qp))"),
    "adamw_no_bias_correction": ("k.step = (float)(h->lr / (1.0 - pow(h->beta1, t)));", "k.step = (float)h->lr;"),
    "adamw_no_eps": ("volatile float den = sc + k->eps;", "volatile float den = sc;"),
    "adamw_no_sqrt": ("volatile float sq = sqrtf(*v);", "volatile float sq = *v;"),
    "adamw_betas_swapped": ("volatile float a1 = k->b1 * *m;", "volatile float a1 = k->b2 * *m;"),
    "adamw_decay_sign": ("k.decay = (float)(1.0 - h->lr * h->weight_decay);", "k.decay = (float)(1.0 + h->lr * h->weight_decay);"),
    "adamw_alpha_uses_w_hparams": ("alpha[r] = pqo_adamw_update(&ka,", "alpha[r] = pqo_adamw_update(&kw,"),
    "reduce_no_multiplier": ("volatile float gbar = sum * grad_mult;", "volatile float gbar = sum;"),
    "reduce_first_source_only": ("volatile float t = sum + pqo_bf16_to_float(g_srcs[k][r * cols + j]);",
                                 "volatile float t = pqo_bf16_to_float(g_srcs[0][r * cols + j]);"),
    "matmul_seq_level": ("else if (p.shift != 0.0f) lev = (2.0 * c + 1.0) / (2.0 * p.kh);",
                         "else if (p.shift != 0.0f) lev = (2.0 * c + 1.0) / 4.0;"),
    "matmul_no_alpha": ("y[i * n + j] = acc * (double)alpha[j];", "y[i * n + j] = acc;"),
    "fwd_level_no_alpha": ("volatile float prod = lev * alpha;",
                         "volatile float prod = lev;"),
    "binary_sign_zero": ("c = (x >= 0.0f) ? 1 : -1;", "c = (x > 0.0f) ? 1 : -1;"),
    "scale_multiplies": ("float x = w / alpha;", "float x = w * alpha;"),
    "seq_level_divisor": ("lev = num / p.kh;", "lev = num / 2.0f;"),
    "ternary_level": ("lev = r / p.kh;", "lev = r / 2.0f;"),
    "zero_sign_dropped": ("c = (int)r;\n    }", "c = (int)r;\n        lev = (lev == 0.0f) ? 0.0f : lev;\n    }"),
    "grad_scale_missing": ("dalpha[r] = (float)(acc * (double)grad_scale);",
                           "dalpha[r] = (float)(acc);"),
    "dequant_no_sign_extend": ("int c = (f & (1u << (p.bits - 1))) ? (int)f - (1 << p.bits) : (int)f;",
                               "int c = (int)f;"),
    "dequant_field_order": ("unsigned f = (byte >> (p.bits * (int)(j % per_byte))) & mask;",
                            "unsigned f = (byte >> (p.bits * (int)(per_byte - 1 - j % per_byte))) & mask;"),
    "dequant_no_alpha": ("volatile float prod = pqo_level_of_code(&p, c) * alpha[r];",
                         "volatile float prod = pqo_level_of_code(&p, c);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(pq_oracle.SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    mutated = src.replace(old, new)
    c_path = os.path.join(tmp_path, "mutant.c")
    so_path = os.path.join(tmp_path, "libmutant.so")
    with open(c_path, "w") as f:
        f.write(mutated)
    pq_oracle.compile_source(c_path, so_path)
    O = pq_oracle.Oracle(so_path)
    failed = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check(O)
        except AssertionError:
            failed.append(check.__name__)
            break
    assert failed, f"mutant {name} passed every pin"
