"""B200-native (sm_100a) fused causal attention, forward and backward."""
from . import workloads  # noqa: F401
