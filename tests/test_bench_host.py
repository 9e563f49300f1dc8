"""Host logic of the benchmark (CPU): both arms describe the workload with
the same config dict, the custom-shape option builds the workload it names,
and the variants switch the right flags."""
import argparse

import pytest

import bench
from mixture_experts_ffn_16_b200.inputs import CONFIGS


def _args(**kw):
    base = dict(shape="", score="softmax", bias_std=0.0, variant="", config="large_imbalanced")
    base.update(kw)
    return argparse.Namespace(**base)


@pytest.mark.parametrize("name", list(CONFIGS))
def test_both_arms_report_the_same_config(name):
    cfg = CONFIGS[name]
    a = bench.config_dict(cfg, "", 1)
    b = bench.config_dict(cfg, "", 1)
    assert a == b and a["workload"] == name
    assert a["T"] == cfg.T and a["E"] == cfg.E and a["k"] == cfg.k and a["d_model"] == cfg.d
    assert a["l2"].startswith("no flush: inputs larger than L2")
    assert bench.config_dict(cfg, "", 8)["parallelism"] == "replicas"


def test_default_workload_is_the_largest(monkeypatch):
    monkeypatch.setattr("sys.argv", ["bench.py"])
    args = bench.parse()
    assert args.config == "large_imbalanced" and args.gpus == 1 and args.warmup >= 3
    sizes = {n: c.T * c.k * 3 * c.f * c.d for n, c in CONFIGS.items()}
    assert max(sizes, key=sizes.get) == "large_imbalanced"


def test_custom_shape():
    cfg = bench.custom_cfg(_args(shape="16384,7168,112,3,512,2,1024", score="sqrt_softplus", bias_std=0.1))
    assert (cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.S, cfg.fs) == (16384, 7168, 112, 3, 512, 2, 1024)
    assert cfg.score_fn == "sqrt_softplus" and cfg.bias_std == 0.1
    assert cfg.name == "custom_T16384_d7168_E112_k3_f512_S2_fs1024"


@pytest.mark.parametrize("variant,flag", [("gated_shared", "shared_gate"), ("prenorm", "prenorm"), ("fp8", "fp8")])
def test_variants(variant, flag):
    cfg = bench.variant_cfg(CONFIGS["prefill_softmax"], variant)
    assert getattr(cfg, flag) is True
    assert bench.config_dict(cfg, variant, 1)["variant"] == variant
    assert bench.variant_cfg(CONFIGS["prefill_softmax"], "") == CONFIGS["prefill_softmax"]
