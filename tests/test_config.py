"""Megatron-Bridge recipe keys -> library arguments (host logic, no GPU)."""

import pytest

from muon_step_b200.config import AGGRESSIVE, HYBRID, STANDARD, MuonConfig, from_megatron

# the DeepSeek-V4-Flash recipe's optimizer keys as the V4 breakdown page prints them
RECIPE = dict(muon_momentum=0.95, muon_use_nesterov=True, muon_scale_mode="unit_rms_norm",
              muon_fp32_matmul_prec="highest", muon_num_ns_steps=5, muon_extra_scale_factor=0.2,
              lr_warmup_iters=2000, max_lr=2.7e-4, min_lr=2.7e-5, weight_decay=0.1, clip_grad=1.0,
              optimizer="muon", muon_coefficient_type="quintic")


def test_recipe_maps_onto_the_library():
    cfg = from_megatron(**RECIPE)
    assert cfg.momentum == 0.95 and cfg.nesterov is True
    assert cfg.scale_mode == "unit_rms" and cfg.gamma == 0.2
    assert cfg.precision == "fp32"
    assert cfg.schedule == (AGGRESSIVE,) * 5
    assert cfg.lr == 2.7e-4 and cfg.weight_decay == 0.1
    assert cfg.unused == {"lr_warmup_iters": 2000, "min_lr": 2.7e-5, "clip_grad": 1.0}
    assert cfg.plan_kwargs() == {"precision": "fp32", "schedule": (AGGRESSIVE,) * 5,
                                 "scale_mode": "unit_rms"}
    assert cfg.execute_kwargs() == {"lr": 2.7e-4, "momentum": 0.95, "weight_decay": 0.1,
                                    "gamma": 0.2, "nesterov": True}


def test_deepseekv4_coefficients_are_the_hybrid_schedule():
    cfg = from_megatron(muon_coefficient_type="deepseekv4", muon_num_ns_steps=10)
    assert cfg.schedule == HYBRID
    assert HYBRID[:8] == (AGGRESSIVE,) * 8 and HYBRID[8:] == (STANDARD,) * 2
    with pytest.raises(ValueError):
        from_megatron(muon_coefficient_type="deepseekv4", muon_num_ns_steps=5)


def test_defaults_and_precision_choice():
    assert from_megatron() == MuonConfig()
    assert from_megatron(muon_fp32_matmul_prec="medium").precision == "bf16"
    assert from_megatron(muon_num_ns_steps=3).schedule == (AGGRESSIVE,) * 3


@pytest.mark.parametrize("bad", [dict(muon_scale_mode="spectral_norm"),
                                 dict(muon_coefficient_type="cubic"),
                                 dict(muon_num_ns_steps=0)])
def test_unknown_values_are_rejected(bad):
    with pytest.raises(ValueError):
        from_megatron(**bad)
