def roofline_time_us(nbytes: float, gbps: float) -> float:
    """Time in microseconds to move ``nbytes`` at ``gbps`` GB/s (1 GB = 1e9 B)."""
    return nbytes / (gbps * 1e9) * 1e6
