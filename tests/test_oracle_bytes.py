"""Byte accounting of the persistent state against the pages' figures (CPU)."""
import json
import os

import pytest

import oracle
from workloads import tensor_list


def _acct(name):
    ts = tensor_list(name)
    o = oracle.OracleAdamW4(tensors=ts)
    q = sum(t.numel for t in o.tensors if not t.fp32)
    f = sum(t.numel for t in o.tensors if t.fp32)
    return o, q, f


def test_per_param_and_reduction(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "byte_accounting.json")))
    o = oracle.OracleAdamW4(tensors=[dict(numel=128 * 1000, tensor_id=0)])
    assert o.state_bytes() / (128 * 1000) == g["quant_bytes_per_param"]
    assert round(g["fp32_bytes_per_param"] / g["quant_bytes_per_param"], 2) == g["reduction"]


def test_wikitext_table_bytes(golden_dir):
    """The 2-layer byte-level GPT reproduces both figures of the table exactly:
    135,168 quantised and 1,792 fp32-state parameters."""
    g = json.load(open(os.path.join(golden_dir, "byte_accounting.json")))
    o, q, f = _acct("microlm-p4")
    assert (q, f) == (135168, 1792)
    assert 8 * (q + f) == g["table_fp32_bytes"]
    assert o.state_bytes() == g["table_4bit_bytes"]
    saving = 100 * (1 - o.state_bytes() / (8 * (q + f)))
    assert round(saving, 1) == g["table_saving_percent"]


def test_2p7b_memory_saved(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "byte_accounting.json")))
    o, q, f = _acct("gpt-2.7b")
    assert q + f == 2780451840
    saved = 8 * (q + f) - o.state_bytes()
    assert saved / 1e9 == pytest.approx(g["saved_gb_2p7b"], abs=0.1)


@pytest.mark.parametrize("name,q,f,n", [("gpt-130m", 124354560, 121344, 148),
                                        ("llama-1.1b", 1099956224, 92160, 201),
                                        ("gpt-2.7b", 2779955200, 496640, 389)])
def test_tensor_lists(name, q, f, n):
    o, qq, ff = _acct(name)
    assert (qq, ff, len(o.tensors)) == (q, f, n)
