"""Synthetic layer workloads shaped like the GPTQ pages' OPT / LLaMA experiments.

Each workload is a list of linear layers (rows = out features, cols = in
features) with the quantizer settings it is run at.  The calibration set is
128 sequences x 2048 tokens (262144 tokens), the size the GPTQ pages use for
their calibration data; the tiny workload uses 2048 tokens.
"""
from __future__ import annotations

from dataclasses import dataclass, field

from .synthetic import BF16, F16, F32, ActSpec, WeightSpec

CALIB_TOKENS = 128 * 2048


@dataclass(frozen=True)
class QuantSetting:
    bits: int = 4
    group_size: int = 128      # 0 = one grid per row
    sym: bool = False
    act_order: bool = False
    damp: float = 0.01
    block_size: int = 128

    def label(self) -> str:
        g = "row" if self.group_size <= 0 else f"g{self.group_size}"
        return f"{self.bits}b-{'sym' if self.sym else 'asym'}-{g}{'-act' if self.act_order else ''}"


@dataclass(frozen=True)
class Layer:
    name: str
    rows: int
    cols: int
    tag: int


@dataclass(frozen=True)
class Workload:
    name: str
    layers: tuple
    wdtype: str
    xdtype: str
    tokens: int
    wspec: WeightSpec
    xspec: ActSpec
    quant: tuple = field(default_factory=tuple)  # one or more QuantSetting


WORKLOADS = {
    "tiny": Workload(
        name="tiny-256x128",
        layers=(Layer("tiny", 256, 128, 1),),
        wdtype=F32, xdtype=F32, tokens=2048,
        wspec=WeightSpec(sigma=0.02),
        xspec=ActSpec(dist="normal", outlier_count=4, outlier_mult=10.0),
        quant=(QuantSetting(bits=4, group_size=0, act_order=False),),
    ),
    "opt125m": Workload(
        name="opt-125m-shaped",
        layers=(Layer("attn.q_proj", 768, 768, 11),
                Layer("fc1", 3072, 768, 12),
                Layer("fc2", 768, 3072, 13)),
        wdtype=F16, xdtype=F16, tokens=CALIB_TOKENS,
        wspec=WeightSpec(sigma=0.02, outlier_frac=0.001, outlier_mult=8.0),
        xspec=ActSpec(dist="t4", outlier_frac=0.01, outlier_mult=20.0),
        quant=(QuantSetting(bits=4, group_size=128),),
    ),
    "llama7b": Workload(
        name="llama-7b-shaped",
        layers=(Layer("self_attn.q_proj", 4096, 4096, 21),
                Layer("mlp.gate_proj", 11008, 4096, 22),
                Layer("mlp.down_proj", 4096, 11008, 23)),
        wdtype=BF16, xdtype=BF16, tokens=CALIB_TOKENS,
        wspec=WeightSpec(sigma=0.02),
        xspec=ActSpec(dist="t4", outlier_frac=0.01, outlier_mult=20.0),
        quant=(QuantSetting(bits=4, group_size=128, act_order=True),),
    ),
    "llama13b": Workload(
        name="llama-13b-shaped",
        layers=(Layer("self_attn.q_proj", 5120, 5120, 31),
                Layer("mlp.gate_proj", 13824, 5120, 32),
                Layer("mlp.down_proj", 5120, 13824, 33)),
        wdtype=F16, xdtype=F16, tokens=CALIB_TOKENS,
        wspec=WeightSpec(sigma=0.02),
        xspec=ActSpec(dist="t4", outlier_frac=0.01, outlier_mult=20.0),
        quant=(QuantSetting(bits=3, group_size=0),
               QuantSetting(bits=2, group_size=64),
               QuantSetting(bits=4, group_size=128, sym=True)),
    ),
    "opt175b": Workload(
        name="opt-175b-shaped",
        layers=(Layer("attn.qkv_proj", 12288, 12288, 41),
                Layer("fc1", 49152, 12288, 42),
                Layer("fc2", 12288, 49152, 43)),
        wdtype=F16, xdtype=F16, tokens=CALIB_TOKENS,
        wspec=WeightSpec(sigma=0.015, outlier_frac=0.0005, outlier_mult=10.0),
        xspec=ActSpec(dist="t4", outlier_frac=0.01, outlier_mult=20.0),
        quant=(QuantSetting(bits=4, group_size=128, act_order=True),),
    ),
}

ORDER = ("tiny", "opt125m", "llama7b", "llama13b", "opt175b")
