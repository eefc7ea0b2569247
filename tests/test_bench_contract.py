"""The benchmark's metric arithmetic (CPU): its parameter counts agree with the oracle's
tensor table and with the counts the pages print, and FLOPs per token follow
6 N + 12 L T C: six per parameter per token for forward and backward, plus the attention
score and value products over the full context."""
import importlib.util
import os

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _golden():
    out = {}
    for line in open(os.path.join(ROOT, "tests", "golden", "page_constants.txt")):
        line = line.split("#", 1)[0].strip()
        if "=" in line:
            k, v = (x.strip() for x in line.split("=", 1))
            out[k] = float(v)
    return out


def test_param_counts_match_oracle_and_pages():
    b = _bench()
    g = _golden()
    for name, c in b.CONFIGS.items():
        oc = oracle.Config(c["L"], c["H"], c["C"], c["T"], c["V"], c["tied"], c["qkv_bias"])
        assert b.n_params(c) == oracle.num_params(oc), name
    assert b.n_params(b.CONFIGS["gpt2-124m"]) == g["param_count_gpt2_124m_tied_v50257"]
    assert b.n_params(b.CONFIGS["gpt2-124m-untied"]) == g["param_count_untied_163m"]


def test_flops_per_token():
    b = _bench()
    c = b.CONFIGS["gpt2-124m"]
    assert b.flops_per_token(c) == 6 * 124_439_808 + 12 * 12 * 1024 * 768 == 859_885_056
