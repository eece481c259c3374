"""Plant a mistake in a copy of the oracle and check that the pins catch it.

Each mutant is the oracle's C source with one plausible slip (a wrong group
map, a dropped term, a wrong sign or index, a transposed operand).  The copy is
compiled on the CPU into a temporary library; the real oracle is untouched.
"""
import functools
import os

import pytest

import oracle
from tests.oracle_pins import LSE_PINS, MAPPED_PINS, PINS, VERIFY_PINS

MUTANTS = {
    "group map i % G": ("const int32_t g = group_of_head ? group_of_head[i] : i / r;",
                        "const int32_t g = group_of_head ? group_of_head[i] : i % G;"),
    "scale dropped": ("logits[t] = scale * dot;", "logits[t] = dot;"),
    "page row index transposed": ("row_in_page = t % page_size;", "row_in_page = t / page_size;"),
    "page table stride": ("page_table[(long long)s * max_pages_per_seq + t / page_size]",
                          "page_table[(long long)s + t / page_size]"),
    "K read as V": ("o[k] += w * bf16_to_f64(v_cache[off + k]);",
                    "o[k] += w * bf16_to_f64(k_cache[off + k]);"),
    "max subtracted with wrong sign": ("logits[t] = exp(logits[t] - mx);",
                                       "logits[t] = exp(mx - logits[t]);"),
    "normaliser dropped": ("const double w = logits[t] / denom;", "const double w = logits[t];"),
    "query row of head 0": ("const uint16_t *qi = q + row * (int64_t)d;",
                            "const uint16_t *qi = q + (int64_t)s * H * d;"),
    "bf16 widened with wrong shift": ("((uint32_t)bits) << 16", "((uint32_t)bits) << 15"),
    "group stride dropped": ("((page * G + g) * (long long)page_size", "((page + g) * (long long)page_size"),
    "last token dropped": ("for (int32_t t = 0; t < len; ++t) {\n            const long long off",
                           "for (int32_t t = 0; t < len - 1; ++t) {\n            const long long off"),
    "capacity check off by one": ("if (len_s < nq || len_s > capacity)", "if (len_s < nq || len_s > capacity + 1)"),
    "draft mask reversed": ("const int32_t len = len_s - (nq - 1 - tq);", "const int32_t len = len_s - tq;"),
    "draft mask off by one": ("const int32_t len = len_s - (nq - 1 - tq);", "const int32_t len = len_s - (nq - tq);"),
    "map read at the next head": ("const int32_t g = group_of_head ? group_of_head[i] : i / r;",
                                  "const int32_t g = group_of_head ? group_of_head[(i + 1) % H] : i / r;"),
    "map of head 0 for every head": ("const int32_t g = group_of_head ? group_of_head[i] : i / r;",
                                     "const int32_t g = group_of_head ? group_of_head[0] : i / r;"),
    "draft index of the row": ("const int32_t tq = (int32_t)((row / H) % nq);", "const int32_t tq = (int32_t)(row % nq);"),
    "page bound off by one": ("if (page < 0 || page >= num_pages)", "if (page < 0 || page > num_pages)"),
    "lse without the maximum": ("lse[n] = mx + log(denom);", "lse[n] = log(denom);"),
    "lse not a logarithm": ("lse[n] = mx + log(denom);", "lse[n] = mx + denom;"),
    "lse of the last logit": ("lse[n] = mx + log(denom);", "lse[n] = logits[len - 1];"),
}


@functools.lru_cache(maxsize=None)
def _source():
    with open(os.path.join(os.path.dirname(oracle.__file__), "gqa_oracle.c")) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = _source()
    assert src.count(old) >= 1, "mutation site not found: %r" % old
    mutated = src.replace(old, new)
    path = tmp_path / "mutant.c"
    path.write_text(mutated)
    lib = oracle.load_library(oracle.build(force=True, src=str(path), out=str(tmp_path / "libmutant.so")))
    decode = functools.partial(oracle.gqa_decode, lib=lib)
    decode_lse = functools.partial(oracle.gqa_decode_lse, lib=lib)
    decode_verify = functools.partial(oracle.gqa_decode_verify, lib=lib)
    decode_mapped = functools.partial(oracle.gqa_decode_mapped, lib=lib)
    caught = []
    for pins, fn in ((PINS, decode), (LSE_PINS, decode_lse), (VERIFY_PINS, decode_verify),
                     (MAPPED_PINS, decode_mapped)):
        for pin in pins:
            try:
                pin(fn)
            except (AssertionError, ValueError, IndexError):
                caught.append(pin.__name__)
    assert caught, "no pin caught the mutant %r" % name
