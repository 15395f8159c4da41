"""The CPU oracle against closed forms, library routines, brute force and the
invariants of "Bifocal Diffusion Language Models" (arXiv 2606.27732v1), §3.4."""
import json
import os

import pytest

import oracle as O
from reverse_selective_ssm_b200 import synthetic as S

from . import pins

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(O)


def test_parameter_count_matches_paper():
    """C0: the block shapes (expand 2, d_state 16, d_conv 4, dt_rank d/16) give
    the 185M extra parameters of Table 4 / §4.2 over 7 hooks, 10.8% of a 1.7B
    backbone (§5).  Counts the tensors the generator draws plus the gate s."""
    facts = json.load(open(os.path.join(HERE, "golden", "paper_facts.json")))
    dims = S.BIG
    assert dims.d_model == facts["d_model"]["value"]
    assert dims.d_state == facts["d_state"]["value"]
    assert dims.d_conv == facts["d_conv"]["value"]
    assert dims.d_inner == facts["expand"]["value"] * dims.d_model
    hooks = facts["decoder_layers"]["value"] // facts["hook_every_k"]["value"]
    assert hooks == facts["hooks"]["value"]
    w = S.make_weights(dims, S.torch.bfloat16, seed=0)
    per_hook = sum(t.numel() for t in w.values() if t is not None) + 1   # + scalar gate s
    assert per_hook == 26_443_777
    total_m = per_hook * hooks / 1e6
    assert abs(total_m - facts["sidecar_params_millions"]["value"]) < 0.5, total_m
    backbone_b = total_m / 1e3 / (facts["sidecar_fraction_of_backbone_percent"]["value"] / 100)
    assert abs(backbone_b - facts["backbone_params_billions"]["value"]) < 0.05, backbone_b
