"""Benchmark of the simulated-rank collectives (filled in below)."""


def busbw_all_reduce(size_bytes: float, p: int, t: float) -> float:
    """Bus bandwidth 2 s (p-1) / (p t) in bytes/s: "分布式训练/推理", section
    "带宽怎么核算：看 duration 之前先看 bytes" (s = bytes of one rank's tensor)."""
    return 2.0 * size_bytes * (p - 1) / (p * t)


def busbw_reduce_scatter(input_bytes: float, p: int, t: float) -> float:
    """Bus bandwidth s_input (p-1) / (p t), same section; s_input is the
    world_size x k input of one rank."""
    return input_bytes * (p - 1) / (p * t)
