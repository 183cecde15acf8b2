"""Planted mistakes: every plausible slip in the oracle must fail at least one pin.

Each case copies oracle/attn_fp64.c, applies one textual mistake (a dropped term, a
wrong sign, an off-by-one mask, a wrong index or head mapping, a transposed operand),
compiles the copy into a temporary library and runs the pin suite against it.  The
mistakes live only in these temporary copies, on the CPU.
"""
import functools
import os
import subprocess

import pytest

import oracle
from tests import pin_suite

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_fp64.c")

MUTANTS = {
    "scale_dropped": ("double sj = J->scale * dot;", "double sj = dot;"),
    "max_sign_flipped": ("double p = exp(s[j] - m);", "double p = exp(m - s[j]);"),
    "max_not_subtracted": ("double p = exp(s[j] - m);", "double p = exp(s[j]);"),
    "no_normalisation": ("o_row[c] = o_row[c] / l;", "o_row[c] = o_row[c];"),
    "lse_without_max": ("*lse = m + log(l);", "*lse = log(l);"),
    "lse_log2": ("*lse = m + log(l);", "*lse = m + log2(l);"),
    "causal_off_by_one": ("if (J->causal && j > pos)", "if (J->causal && j >= pos)"),
    "causal_local_index": ("if (J->causal && j > pos)", "if (J->causal && j > i)"),
    "window_off_by_one": ("pos - j >= J->window", "pos - j > J->window"),
    "softcap_inner_scale_dropped": ("tanh(sj / J->softcap)", "tanh(sj)"),
    "softcap_outer_scale_dropped": ("sj = J->softcap * tanh(sj / J->softcap);", "sj = tanh(sj / J->softcap);"),
    "gqa_modulo_mapping": ("const int64_t kv = hq / group;", "const int64_t kv = hq % J->Hkv;"),
    "value_row_is_query_row": ("p * load_elem(J->v, J->dtype, kv_base + j * d + c)",
                               "p * load_elem(J->v, J->dtype, kv_base + (j < N - 1 ? j + 1 : j) * d + c)"),
    "keys_used_as_values": ("p * load_elem(J->v, J->dtype, kv_base + j * d + c)",
                            "p * load_elem(J->k, J->dtype, kv_base + j * d + c)"),
    "queries_used_as_keys": ("load_elem(J->k, J->dtype, kv_base + j * d + c);",
                             "load_elem(J->q, J->dtype, ((b * J->Hq + hq) * Nq + (j < Nq ? j : 0)) * d + c);"),
    "last_key_dropped": ("for (int64_t j = 0; j < N; ++j) {\n    double p", "for (int64_t j = 0; j + 1 < N; ++j) {\n    double p"),
    "sum_without_first_key": ("    l += p;", "    if (j) l += p;"),
    "sinks_ignored": (" && j >= J->n_sink) sj", ") sj"),
    "sinks_off_by_one": ("j >= J->n_sink", "j > J->n_sink"),
    "sinks_override_causal": ("if (J->causal && j > pos)", "if (J->causal && j > pos && j >= J->n_sink)"),
    "sinks_without_window": ("if (J->window > 0 && pos - j >= J->window && j >= J->n_sink)",
                             "if ((J->window > 0 && pos - j >= J->window) || (J->n_sink > 0 && j >= J->n_sink))"),
    "cross_top_left_causal": ("const int64_t pos = i + (N - Nq);", "const int64_t pos = i;"),
    # widening of the stored bf16 bits (the top half of an IEEE binary32)
    "bf16_shift_by_15": ("((const uint16_t*)base)[idx] << 16;", "((const uint16_t*)base)[idx] << 15;"),
    "bf16_low_half": ("((const uint16_t*)base)[idx] << 16;", "((const uint16_t*)base)[idx];"),
    "bf16_byte_swap": ("((const uint16_t*)base)[idx] << 16;",
                       "(uint16_t)((((const uint16_t*)base)[idx] >> 8) | (((const uint16_t*)base)[idx] << 8)) << 16;"),
    "bf16_sign_dropped": ("((const uint16_t*)base)[idx] << 16;", "(((const uint16_t*)base)[idx] & 0x7FFFu) << 16;"),
}


@pytest.fixture(scope="module")
def mutant_dir(tmp_path_factory):
    """One pytest-managed temporary directory for the mutant builds of this module."""
    return str(tmp_path_factory.mktemp("oracle_mutants"))


def _build_mutant(name, directory):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    c_path = os.path.join(directory, f"{name}.c")
    so_path = os.path.join(directory, f"lib{name}.so")
    open(c_path, "w").write(src.replace(old, new))
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-pthread", c_path, "-o", so_path, "-lm"],
                   check=True)
    return oracle.load_library(so_path)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(name, mutant_dir):
    lib = _build_mutant(name, mutant_dir)
    attn = functools.partial(oracle.attention, _lib=lib)
    failed = pin_suite.failures(attn)
    assert failed, f"planted mistake {name!r} passed every pin"


def test_bf16_marshalling_mistake_fails_a_pin(monkeypatch):
    """The Python side hands bf16 tensors to the C oracle as raw 16-bit patterns; handing
    over the fp16 patterns of the same values instead (a plausible slip) must fail."""
    import numpy as np
    import torch

    real = oracle._as_host_array

    def fp16_bits(t):
        if isinstance(t, torch.Tensor) and t.dtype == torch.bfloat16:
            h = t.detach().cpu().contiguous().to(torch.float16)
            return h.view(torch.int16).numpy().view(np.uint16), oracle.DTYPE_CODES["bfloat16"]
        return real(t)

    monkeypatch.setattr(oracle, "_as_host_array", fp16_bits)
    with pytest.raises(AssertionError):
        pin_suite.pin_bf16_inputs(oracle.attention)
