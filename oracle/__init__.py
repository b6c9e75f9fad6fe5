"""CPU oracle of the PagedAttention hot path (fp64, plain C + ctypes).  Test infrastructure only."""
