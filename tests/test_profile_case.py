"""The small-case profiling driver checks its arguments before it touches the
GPU (no GPU needed here)."""
import pytest


def test_rejects_fewer_experts_than_k():
    from mixture_experts_topk_b200 import profile_case
    with pytest.raises(SystemExit, match="at least the workload's k"):
        profile_case.main(["--workload", "deepseek-v3", "--experts", "4", "--tokens", "16"])


def test_unknown_workload_is_an_argument_error():
    from mixture_experts_topk_b200 import profile_case
    with pytest.raises(SystemExit):
        profile_case.main(["--workload", "no-such-layer", "--experts", "8", "--tokens", "16"])
