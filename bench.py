"""Benchmark of one denoising step (filled in with the CUDA path)."""


def roofline_seconds(bytes_moved: float, flops: float, hbm_bps: float,
                     flops_per_s: float) -> float:
    """Lower bound on a kernel's time: the slower of moving its bytes at the
    memory bandwidth and doing its FLOPs at the arithmetic peak."""
    return max(bytes_moved / hbm_bps, flops / flops_per_s)
