"""Plausible mistakes planted in a copy of the numpy oracle fail the pins.

Each mutant is the numpy oracle's source with one textual change, executed in
a fresh namespace on the CPU.  The real oracle passes every check in
``pins.ALL_CHECKS``; every mutant must fail at least one, which shows that the
pins would catch that kind of error in the oracle.
"""
import inspect
import types

import numpy as np
import pytest

from oracle import oracle as O
import pins

MUTANTS = {
    # KV head hq % Hkv instead of hq // G
    "head_mapping": ("np.repeat(kc, group, axis=1)", "np.tile(kc, (1, group, 1))"),
    "dropped_scale": ("s = scale * np.einsum", "s = np.einsum"),
    "scale_squared": ("s = scale * np.einsum", "s = scale * scale * np.einsum"),
    "last_token_dropped": ("t = np.arange(ctx)", "t = np.arange(max(ctx - 1, 0))"),
    "block_and_offset_swapped": ("[t // bs], t % bs]", "[t % bs], t // bs]"),
    "keys_used_as_values": ('np.einsum("ht,thd->hd", p, vq)', 'np.einsum("ht,thd->hd", p, kq)'),
    "normalised_over_all_heads": ("/ p.sum(axis=1, keepdims=True)", "/ p.sum()"),
    "no_max_subtraction": ("np.exp(s - s.max(axis=1, keepdims=True))", "np.exp(s)"),
    "sign_flipped_logits": ("np.exp(s - s.max(axis=1, keepdims=True))",
                            "np.exp(-s + s.min(axis=1, keepdims=True))"),
    "query_transposed_heads": ('np.einsum("hd,thd->ht", qf[b], kq)',
                               'np.einsum("hd,thd->ht", qf[b][::-1], kq)'),
}


def _mutant(name):
    old, new = MUTANTS[name]
    src = inspect.getsource(O.paged_attention_np) + "\n" + inspect.getsource(O.gather_np)
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    ns = dict(vars(O))
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), ns)
    return ns["paged_attention_np"]


def _failures(attn):
    failed = []
    for check in pins.ALL_CHECKS:
        try:
            with np.errstate(all="ignore"):
                check(attn)
        except (AssertionError, ValueError, IndexError, FloatingPointError):
            failed.append(check.__name__)
    return failed


def test_unmutated_oracle_passes_every_pin():
    assert _failures(O.paged_attention_np) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_fails_a_pin(name):
    failed = _failures(_mutant(name))
    assert failed, f"mutant {name} passed every pin"
