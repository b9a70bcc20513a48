"""The oracle's pins must catch plausible mistakes.

Each case below compiles a copy of oracle/gdr_oracle.c with one deliberate
mistake (a dropped term, a wrong sign, a wrong operand or index, a wrong order)
and checks that at least one pin rejects it. The mistakes are planted in a
temporary copy of the CPU oracle only.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
from test_oracle_pins import GEN, rand_inputs, read_golden

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdr_oracle.c")

DECAY_BLOCK = """        /* decay: S <- Diag(alpha_t) S */
        for (int i = 0; i < dk; ++i) {
            double a = gate_at(alpha, alpha_pc, tok, dk, i, 1.0);
            for (int j = 0; j < dv; ++j) S[i * dv + j] *= a;
        }
"""
READ_MARK = "        /* read: o_t = q_t S_t */\n"

MUTANTS = {
    "no_decay": [("S[i * dv + j] *= a;", "S[i * dv + j] *= 1.0;")],
    "erase_sign": [("+= -kt[i] * r[j]", "+= kt[i] * r[j]")],
    "erase_read_ignores_b": [("double bk = gate_at(b, b_pc, tok, dk, i, 0.0) * kt[i];",
                              "double bk = kt[i];")],
    "erase_sides_swapped": [("double bk = gate_at(b, b_pc, tok, dk, i, 0.0) * kt[i];",
                             "double bk = kt[i];"),
                            ("+= -kt[i] * r[j]", "+= -gate_at(b, b_pc, tok, dk, i, 0.0) * kt[i] * r[j]")],
    "write_ignores_w": [("double wk = gate_at(w, w_pc, tok, dk, i, 1.0) * kt[i];", "double wk = kt[i];")],
    "no_erase": [("+= -kt[i] * r[j] + wk * vt[j]", "+= wk * vt[j]")],
    "decay_after_update": [(DECAY_BLOCK, ""), (READ_MARK, DECAY_BLOCK + READ_MARK)],
    "channel_gate_index": [("return per_channel ? g[tok * dk + i] : g[tok];",
                            "return per_channel ? g[tok * dk] : g[tok];")],
    "read_with_k": [("ot[j] += qt[i] * S[i * dv + j];", "ot[j] += kt[i] * S[i * dv + j];")],
    "ignores_S0": [("if (S0) memcpy(", "if (0) memcpy(")],
    "value_index_lag": [("const double* vt = v + tok * dv;",
                         "const double* vt = v + (t > 0 ? tok - H : tok) * dv;")],
}


def _pins_pass(lib) -> bool:
    """True if every pin accepts `lib`."""
    ok = True
    g = read_golden("worked_example_dk2_dv3.txt")
    sh = lambda x, d: x.reshape(1, 2, 1, d)
    o, ST = oracle.recurrence(sh(g["q"], 2), sh(g["k"], 2), sh(g["v"], 3), sh(g["alpha"], 2),
                              sh(g["b"], 2), sh(g["w"], 2), g["S0"].reshape(1, 1, 2, 3), GEN, lib=lib)
    ok &= np.array_equal(o.reshape(-1), g["o"]) and np.array_equal(ST.reshape(-1), g["S2"])
    rng = np.random.default_rng(11)
    q, k, v, a, b, w, S0 = rand_inputs(rng, 1, 8, 2, 4, 3, GEN, s0=True, k_unit=False)
    o, ST = oracle.recurrence(q, k, v, a, b, w, S0, GEN, lib=lib)
    ou, STu = oracle.unrolled_contributions(q, k, v, a, b, w, S0, GEN)
    ok &= np.allclose(o, ou, atol=1e-12) and np.allclose(ST, STu, atol=1e-12)
    gates = {"alpha": "channel", "b": "none", "w": "channel"}
    o, _ = oracle.recurrence(q, k, v, a, None, w, None, gates, lib=lib)
    ok &= np.allclose(o, oracle.masked_matrix(q, k, v, a, w, gates), atol=1e-12)
    return bool(ok)


def _build_variant(tmp_path, name, edits):
    src = open(SRC).read()
    for old, new in edits:
        assert old in src, f"mutation {name}: pattern not found"
        src = src.replace(old, new, 1)
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(src)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(c)], check=True)
    return oracle.load_library(str(so))


def test_unmodified_oracle_passes_pins(tmp_path):
    assert _pins_pass(_build_variant(tmp_path, "clean", []))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(tmp_path, name):
    assert not _pins_pass(_build_variant(tmp_path, name, MUTANTS[name]))


# Mistakes planted in the backward pass (gdr_oracle_backward); the pins are the
# finite-difference and closed-form checks of test_oracle_bwd_pins.py.
BWD_MUTANTS = {
    "bwd_dq_from_previous_state": [("acc += St[i * dv + j] * dot[j];", "acc += Sp[i * dv + j] * dot[j];")],
    "bwd_drops_erase_term": [("double dsd = G[i * dv + j] + e * dr[j];", "double dsd = G[i * dv + j];")],
    "bwd_dalpha_decayed_state": [("dal += dsd * Sp[i * dv + j];", "dal += dsd * Sd[i * dv + j];")],
    "bwd_state_grad_not_decayed": [("G[i * dv + j] = a * dsd;", "G[i * dv + j] = dsd;")],
    "bwd_dk_sign": [("dk_out[tok * dk + i] = -acck;", "dk_out[tok * dk + i] = acck;")],
    "bwd_gates_swapped_in_dk": [("+= bi_ * de[i] + wi * du[i];", "+= wi * de[i] + bi_ * du[i];")],
    "bwd_dv_key_without_w": [("accv += u * G[i * dv + j];", "accv += kt[i] * G[i * dv + j];")],
    "bwd_dr_sign": [("dr[j] = -accr;", "dr[j] = accr;")],
    "bwd_drops_write_key_grad": [("accu += G[i * dv + j] * vt[j];", "accu += 0.0 * vt[j];")],
}


def _bwd_pins_pass(lib) -> bool:
    from test_oracle_bwd_pins import fd_mismatch
    ok = fd_mismatch({"alpha": "channel", "b": "channel", "w": "channel"}, True, True, 7, lib=lib) < 1e-7
    ok &= fd_mismatch({"alpha": "scalar", "b": "scalar", "w": "scalar"}, False, False, 8, lib=lib) < 1e-7
    return bool(ok)


def test_unmodified_backward_passes_pins(tmp_path):
    assert _bwd_pins_pass(_build_variant(tmp_path, "clean_bwd", []))


@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_backward_pins_reject_mutant(tmp_path, name):
    assert not _bwd_pins_pass(_build_variant(tmp_path, name, BWD_MUTANTS[name]))
