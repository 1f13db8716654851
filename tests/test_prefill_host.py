"""Host-side checks of the MLA-form prefill module (no GPU): an empty prompt launches nothing and
returns its output untouched; arguments the prefill cannot serve are refused before any launch."""

import pytest
import torch

from latent_attention_decode_tpla_b200 import prefill, tpla


def _dims(maxp=2):
    return tpla.make_dims(B=1, H=8, L=64, R=16, dv=32, g=2, max_pages_per_seq=maxp, num_pages=4, softmax_scale=0.1)


def _args(T):
    bf = torch.bfloat16
    return (torch.zeros(T, 64, dtype=bf), torch.zeros(T, 16, dtype=bf), torch.zeros(T, 8, 64, dtype=bf),
            torch.zeros(T, 8, 16, dtype=bf))


def test_empty_prompt_launches_nothing():
    x, k, q, qp = _args(0)
    out = torch.empty(0, 8, 32)
    assert prefill.mla_prefill(_dims(), x, k, q, qp, None, 1, None, None, 1e-6, torch.zeros(2, dtype=torch.int32),
                               None, None, out) is out


def test_prompt_longer_than_its_pages_is_refused():
    x, k, q, qp = _args(129)                       # 129 tokens need 3 pages, the sequence has 2
    with pytest.raises(ValueError):
        prefill.mla_prefill(_dims(2), x, k, q, qp, None, 1, None, None, 1e-6, torch.zeros(2, dtype=torch.int32),
                            None, None, torch.empty(129, 8, 32))
    with pytest.raises(ValueError):
        prefill.mla_prefill(_dims(4), x, k, q, qp, None, 1, None, None, 1e-6, torch.zeros(4, dtype=torch.int32),
                            None, None, torch.empty(129, 8, 32), chunk=0)
