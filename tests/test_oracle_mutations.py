"""The oracle's pins must catch plausible mistakes.

Each case compiles a copy of the oracle's C source with one deliberate slip
(on the CPU, into a temporary directory) and checks that the brute-force
comparison used by the pins rejects it.
"""
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle
from mla_paged_latent_decode_b200 import synth
from test_oracle_pins import brute_force

SRC = os.path.join(os.path.dirname(oracle.__file__), "mla_oracle.c")

MUTATIONS = {
    "rope_dims_dropped": ("for (int c = 0; c < ORACLE_DQK; ++c) dot +=",
                          "for (int c = 0; c < ORACLE_DV; ++c) dot +="),
    "page_index_ignored": ("block_table[(int64_t)i * bt_stride + t / ORACLE_PAGE]",
                           "block_table[(int64_t)i * bt_stride]"),
    "row_in_page_wrong": ("(page * ORACLE_PAGE + t % ORACLE_PAGE)",
                          "(page * ORACLE_PAGE + t / ORACLE_PAGE)"),
    "causal_off_by_one": ("causal ? L - s_q + j + 1 : L", "causal ? L - s_q + j : L"),
    "value_from_wrong_dims": ("out_row[c] += w * bf16_to_double(v[c])",
                              "out_row[c] += w * bf16_to_double(v[c + 64])"),
    "not_normalised": ("out_row[c] /= l;", "out_row[c] /= 1.0;"),
    "lse_wrong_base": ("return m + log(l);", "return m + log2(l);"),
    "scale_not_applied": ("s[t] = scale * dot;", "s[t] = dot;"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_reject_mutation(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor missing: {old}"
    mutated = src.replace(old, new)
    cfile = tmp_path / "mut.c"
    cfile.write_text(mutated)
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(cfile), "-lm"],
                   check=True)
    lib = oracle.load_library(str(so))
    w = synth.custom_workload(3, 2, 4, [1, 130, 70], causal=True)
    inp = synth.make_inputs(w, seed=21)
    out, lse = oracle.decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens, inp.scale,
                             inp.causal, lib=lib)
    ref_out, ref_lse = brute_force(inp)
    ok_out = np.allclose(out, ref_out, rtol=1e-12, atol=1e-14)
    ok_lse = np.allclose(lse, ref_lse, rtol=1e-12, atol=1e-14, equal_nan=False)
    assert not (ok_out and ok_lse), f"mutation {name} went undetected"
