"""Layer shapes and input recipes of the routed MoE FFN workloads.

Plain data only: every field is a shape, a format tag or a distribution
parameter.  Both the CUDA path and the oracle read these, so nothing here
computes any step of the layer.

Shapes follow the model contracts listed in the LightMoE README ("Compatibility"
table: Qwen3.5-35B-A3B 2048/512 with 256 experts top-8, GLM-5.2 6144/2048 with
256 experts top-8) and the workloads the pages name: Mixtral-8x7B (pure-Triton
fused MoE article) and DeepSeek-V3 (Aleph Alpha inference-model article).
"""
from dataclasses import dataclass, field

# activation / weight / hidden quantisation formats
FMT_FP8_ROW = 0       # e4m3, fp32 scale per weight output channel and per token
FMT_FP8_BLOCK128 = 1  # e4m3, fp32 scale per 128x128 weight block and 1x128 activation block
FMT_NVFP4 = 2         # e2m1, e4m3 scale per 16-element block, fp32 global scale per tensor

SCORE_SOFTMAX = 0     # softmax over the selected k logits
SCORE_SIGMOID = 1     # sigmoid of the selected k logits, normalised to sum 1

# gated activation of the expert MLP, h = act(gate, up)
ACT_SWIGLU = 0          # silu(g) u
ACT_SWIGLU_BOUNDED = 1  # silu(min(g, L)) clamp(u, -L, L)
ACT_SWIGLU_OAI = 2      # g' sigmoid(alpha g') (u' + 1), g' = min(g, L), u' = clamp(u, -L, L)
ACT_GEGLU = 3           # gelu(g) u (erf form)
ACT_REGLU = 4           # relu(g) u
ACT_RELU2 = 5           # relu(u)^2, experts without a gate projection


@dataclass(frozen=True)
class Workload:
    name: str
    H: int
    I: int
    E: int
    k: int
    score: int
    fmt: int
    tokens: tuple
    router_init: str            # "normal" (N(0,1/H)) or "uniform" (U(-sqrt(3/H), sqrt(3/H)))
    zipf_s: float = 0.0         # per-expert router bias exponent; 0 = no bias
    hidden_global_scale: float = 0.0   # static NVFP4 hidden scale (checkpoint-style input)
    act: int = ACT_SWIGLU
    act_alpha: float = 0.0
    act_limit: float = 0.0
    notes: str = ""

    @property
    def has_bias(self):
        return self.zipf_s > 0.0


WORKLOADS = {
    "tiny": Workload("tiny", H=256, I=128, E=8, k=2, score=SCORE_SOFTMAX,
                     fmt=FMT_FP8_ROW, tokens=(16,), router_init="normal"),
    "mixtral-8x7b": Workload("mixtral-8x7b", H=4096, I=14336, E=8, k=2,
                             score=SCORE_SOFTMAX, fmt=FMT_FP8_ROW,
                             tokens=(1, 32, 128, 512, 4096), router_init="uniform"),
    "qwen3.5-35b-a3b": Workload("qwen3.5-35b-a3b", H=2048, I=512, E=256, k=8,
                                score=SCORE_SOFTMAX, fmt=FMT_FP8_ROW,
                                tokens=(64, 8192), router_init="normal", zipf_s=1.2),
    "deepseek-v3": Workload("deepseek-v3", H=7168, I=2048, E=256, k=8,
                            score=SCORE_SIGMOID, fmt=FMT_FP8_BLOCK128,
                            tokens=(16, 4096), router_init="uniform"),
    "glm-5.2": Workload("glm-5.2", H=6144, I=2048, E=256, k=8, score=SCORE_SOFTMAX,
                        fmt=FMT_NVFP4, tokens=(8192,), router_init="normal", zipf_s=1.0,
                        hidden_global_scale=2.0 ** -5),
}


def custom(name="custom", **kw):
    """A workload with explicit fields (tests use small shapes of each format)."""
    base = dict(score=SCORE_SOFTMAX, fmt=FMT_FP8_ROW, tokens=(16,), router_init="normal")
    base.update(kw)
    if base["fmt"] == FMT_NVFP4 and not base.get("hidden_global_scale"):
        base["hidden_global_scale"] = 2.0 ** -5
    return Workload(name=name, **base)
