"""libbdscan: the block-diffusion bidirectional Mamba-2 scan on B200 (sm_100a).

``bidirectional_mamba_state_b200.bdscan`` is the Python binding of the C-ABI
library (argument marshalling only); ``workload`` draws seeded inputs.
"""
